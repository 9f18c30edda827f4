"""Plain float64 definition of every step of the encoder forward pass.

Test infrastructure only (see the package docstring).  Citations name the
page and its section; [MOSS] is the MOSS-Transcribe-preview-2B-GGUF model
card, [CW] the CrisperWhisper ONNX-export page.

Where the pages leave a step open, the reading taken is stated at the
function.  Pins (in tests/test_oracle_*.py) for each function:

  hann_periodic, power_spectrum  numpy.fft.rfft on random frames; one-sided
                                 Parseval; a bin-centred cosine keeps its
                                 energy in bins k0-1..k0+1
  mel_filterbank                 torchaudio melscale_fbanks (slaney/slaney)
  log_mel                        transformers WhisperFeatureExtractor (the
                                 routine [MOSS] Architecture "Audio" names);
                                 frame count n/160; silent-frame invariant
  conv2d, conv1d                 torch conv2d / conv1d in float64
  attention_windows              == attention_masked (explicit -inf mask)
                                 == torch scaled_dot_product_attention fp64
  layer_norm, gelu, silu         torch layer_norm / gelu / silu in float64
  sinusoids                      closed forms: PE[0], |PE[p]|^2 = d/2, the
                                 first and last frequency columns
  encoder (1-2 tiny layers),
  head, adapter                  float64 torch composition of library ops
  token_count, window_partition  closed forms 13 n/16000 and n/320, and
                                 ceil(T/104) windows per clip
  splice_embeddings              a hand-written prompt whose spliced rows are
                                 listed explicitly in the test
  encode_stream                  == encode_clip for a stream of one window;
                                 longer streams vs a float64 torch
                                 composition (torch.stft, torchaudio
                                 filterbank, per-window normalisation)
Parity unpinned: the per-chunk position reading (pos_mode 0) and the
channel-major flatten before conv_out are conventions that only trained
weights could distinguish; they are fixed by reading, not by a pin.
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import erf

__all__ = [
    "hann_periodic", "frame_signal", "power_spectrum", "hz_to_mel_slaney", "mel_to_hz_slaney",
    "mel_filterbank", "log_mel", "conv2d", "conv1d", "gelu", "silu", "layer_norm", "sinusoids",
    "linear", "token_count", "window_partition", "attention_windows", "attention_masked", "window_mask",
    "encoder_layer", "stem_conv2d_chunked", "stem_conv1d", "encode_tokens", "encode_clip", "forward",
    "as64", "splice_embeddings", "encode_stream",
]

SAMPLE_RATE = 16000


def as64(t) -> np.ndarray:
    """Weights arrive as torch tensors (bf16 or fp32); upcast exactly to fp64."""
    try:
        import torch
        if isinstance(t, torch.Tensor):
            return t.detach().to(torch.float64).cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(t, dtype=np.float64)


# --------------------------------------------------------------------------
# Log-mel front-end.  [MOSS] Architecture, "Audio" row: 16 kHz mono, 128 mel
# bins, n_fft=400, hop=160, matching WhisperFeatureExtractor; Implementation
# notes: mel compared as "C++ STFT vs WhisperFeatureExtractor"; gotchas: the
# trailing STFT frame is dropped so that there are n_samples/hop frames.
# --------------------------------------------------------------------------

def hann_periodic(n_fft: int) -> np.ndarray:
    """Periodic Hann window w[n] = 0.5 - 0.5 cos(2 pi n / N), n = 0..N-1.

    Reading: periodic (not symmetric), the window WhisperFeatureExtractor
    applies ([MOSS] Architecture, "Audio" row names it as the definition).
    """
    n = np.arange(n_fft, dtype=np.float64)
    return 0.5 - 0.5 * np.cos(2.0 * math.pi * n / n_fft)


def frame_signal(pcm: np.ndarray, n_fft: int, hop: int) -> np.ndarray:
    """Centred framing: reflect-pad n_fft/2 samples on each side, then frames
    f = 0 .. n/hop, frame f covering padded samples [f*hop, f*hop + n_fft).

    Reading: centre=True with reflect padding, the only framing that yields
    exactly n_samples/hop frames once the trailing frame is dropped ([MOSS]
    Non-obvious gotchas, trailing-frame item).
    """
    x = np.asarray(pcm, dtype=np.float64)
    pad = n_fft // 2
    if x.shape[0] <= pad:
        raise ValueError("reflect padding needs more than n_fft/2 samples")
    xp = np.concatenate([x[pad:0:-1], x, x[-2:-pad - 2:-1]])
    n_frames = 1 + (xp.shape[0] - n_fft) // hop
    idx = np.arange(n_fft)[None, :] + hop * np.arange(n_frames)[:, None]
    return xp[idx]


def power_spectrum(pcm: np.ndarray, n_fft: int = 400, hop: int = 160) -> np.ndarray:
    """|X_f[k]|^2 for k = 0..n_fft/2, trailing frame dropped -> [n/hop, n_fft/2+1].

    X_f[k] = sum_n w[n] x_f[n] exp(-2 pi i k n / N), written out as the dense
    DFT (a matrix product with the cos / sin tables).  Power, not magnitude:
    the WhisperFeatureExtractor definition.  The dropped trailing frame is
    [MOSS] Non-obvious gotchas ("stft[..., :-1]").
    """
    frames = frame_signal(pcm, n_fft, hop) * hann_periodic(n_fft)[None, :]
    n = np.arange(n_fft, dtype=np.float64)
    k = np.arange(n_fft // 2 + 1, dtype=np.float64)
    ang = 2.0 * math.pi * np.outer(n, k) / n_fft
    re = frames @ np.cos(ang)
    im = -(frames @ np.sin(ang))
    p = re * re + im * im
    return p[:-1]


def hz_to_mel_slaney(f):
    """Slaney mel scale: linear 3 f / 200 below 1 kHz, logarithmic above with
    27 / ln(6.4) mels per natural-log unit (the scale WhisperFeatureExtractor
    builds its 'slaney' filters on)."""
    f = np.asarray(f, dtype=np.float64)
    f_sp = 200.0 / 3.0
    min_log_hz = 1000.0
    min_log_mel = min_log_hz / f_sp
    logstep = math.log(6.4) / 27.0
    lin = f / f_sp
    with np.errstate(divide="ignore", invalid="ignore"):
        logpart = min_log_mel + np.log(np.maximum(f, 1e-300) / min_log_hz) / logstep
    return np.where(f >= min_log_hz, logpart, lin)


def mel_to_hz_slaney(m):
    m = np.asarray(m, dtype=np.float64)
    f_sp = 200.0 / 3.0
    min_log_hz = 1000.0
    min_log_mel = min_log_hz / f_sp
    logstep = math.log(6.4) / 27.0
    return np.where(m >= min_log_mel, min_log_hz * np.exp(logstep * (m - min_log_mel)), f_sp * m)


def mel_filterbank(n_freqs: int = 201, n_mels: int = 128, sr: int = SAMPLE_RATE,
                   f_min: float = 0.0, f_max: float = 8000.0) -> np.ndarray:
    """Slaney filterbank [n_freqs, n_mels].

    n_mels + 2 points uniform on the Slaney mel scale between f_min and f_max;
    filter i is the triangle rising from point i to point i+1 and falling to
    point i+2, evaluated at the FFT bin frequencies k * sr / n_fft, and scaled
    by 2 / (f_{i+2} - f_i) (Slaney area normalisation).  [MOSS] Architecture,
    "Audio" row: 128 bins matching WhisperFeatureExtractor (80 for the
    whisper-small geometry of [CW]).
    """
    fft_freqs = np.linspace(0.0, sr / 2.0, n_freqs)
    m_pts = np.linspace(hz_to_mel_slaney(f_min), hz_to_mel_slaney(f_max), n_mels + 2)
    f_pts = mel_to_hz_slaney(m_pts)
    fb = np.zeros((n_freqs, n_mels), dtype=np.float64)
    for i in range(n_mels):
        lo, ce, hi = f_pts[i], f_pts[i + 1], f_pts[i + 2]
        up = (fft_freqs - lo) / (ce - lo)
        down = (hi - fft_freqs) / (hi - ce)
        fb[:, i] = np.maximum(0.0, np.minimum(up, down)) * (2.0 / (hi - lo))
    return fb


def log_mel(pcm: np.ndarray, n_mels: int = 128, n_fft: int = 400, hop: int = 160,
            floor: float = 1e-10) -> np.ndarray:
    """Log-mel spectrogram of one clip, [n_mels, n/hop].

    mel = P @ fb; L = log10(max(mel, floor)); m = max over the whole clip;
    L = max(L, m - 8); out = (L + 4) / 4.  This is the WhisperFeatureExtractor
    normalisation named by [MOSS] Architecture, "Audio" row.
    Readings: the floor 1e-10 only guards log(0) (any floor below 10^(m-8)
    gives the same output); the max is per clip, over all bins and frames.
    """
    p = power_spectrum(pcm, n_fft, hop)
    fb = mel_filterbank(n_fft // 2 + 1, n_mels)
    mel = p @ fb                                   # [F, M]
    lg = np.log10(np.maximum(mel, floor))
    lg = np.maximum(lg, lg.max() - 8.0)
    return ((lg + 4.0) / 4.0).T


# --------------------------------------------------------------------------
# Convolutions and element-wise functions.
# --------------------------------------------------------------------------

def conv2d(x: np.ndarray, w: np.ndarray, b, stride: int = 2, pad: int = 1) -> np.ndarray:
    """out[o, i, j] = b[o] + sum_{c, u, v} w[o, c, u, v] * xp[c, s i + u, s j + v],
    xp = x zero-padded by ``pad`` on both spatial axes.  x: [C_in, H, W].

    [MOSS] Architecture, "Conv front-end": 3 x Conv2D stride 2.  Kernel 3 and
    padding 1 are the reading that maps 128 mel bins to the 16 of 480*16.
    The sum over taps (u, v) is written out; the sum over c is a matmul.
    """
    c_in, h, wd = x.shape
    c_out, _, kh, kw = w.shape
    xp = np.zeros((c_in, h + 2 * pad, wd + 2 * pad), dtype=np.float64)
    xp[:, pad:pad + h, pad:pad + wd] = x
    ho = (h + 2 * pad - kh) // stride + 1
    wo = (wd + 2 * pad - kw) // stride + 1
    out = np.zeros((c_out, ho, wo), dtype=np.float64)
    for u in range(kh):
        for v in range(kw):
            patch = xp[:, u:u + stride * (ho - 1) + 1:stride, v:v + stride * (wo - 1) + 1:stride]
            out += np.einsum("oc,chw->ohw", w[:, :, u, v], patch, optimize=True)
    if b is not None:
        out += np.asarray(b, dtype=np.float64)[:, None, None]
    return out


def conv1d(x: np.ndarray, w: np.ndarray, b, stride: int = 1, pad: int = 1) -> np.ndarray:
    """out[o, i] = b[o] + sum_{c, u} w[o, c, u] * xp[c, s i + u]; x: [C_in, T].

    [CW] What this exports instead: whisper-small geometry, whose stem is
    Conv1D k3 s1 then Conv1D k3 s2; padding 1 on both is the reading that
    gives the 1500 encoder frames of [CW] Results.
    """
    c_in, t = x.shape
    c_out, _, k = w.shape
    xp = np.zeros((c_in, t + 2 * pad), dtype=np.float64)
    xp[:, pad:pad + t] = x
    to = (t + 2 * pad - k) // stride + 1
    out = np.zeros((c_out, to), dtype=np.float64)
    for u in range(k):
        out += w[:, :, u] @ xp[:, u:u + stride * (to - 1) + 1:stride]
    if b is not None:
        out += np.asarray(b, dtype=np.float64)[:, None]
    return out


def gelu(x):
    """Exact GELU, x * Phi(x) = 0.5 x (1 + erf(x / sqrt 2)).  Reading: the
    pages say "GELU" without qualification; the erf form is taken."""
    return 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))


def silu(x):
    """SiLU x * sigmoid(x), the gate of the SwiGLU adapter ([MOSS] Architecture,
    "Adapter" row)."""
    return x / (1.0 + np.exp(-x))


def layer_norm(x: np.ndarray, g, b, eps: float = 1e-5) -> np.ndarray:
    """LayerNorm over the last axis: two-pass mean and biased variance.
    [MOSS] Architecture, "Audio encoder": pre-LN Transformer."""
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * np.asarray(g, np.float64) + np.asarray(b, np.float64)


def sinusoids(length: int, d: int, max_timescale: float = 10000.0) -> np.ndarray:
    """Sinusoidal positions [length, d]: d/2 frequencies
    inv_i = exp(-ln(max_timescale) * i / (d/2 - 1)), PE[p] = [sin(p inv), cos(p inv)].
    [MOSS] Architecture, "Conv front-end": "sinusoidal positions".  The pages
    give no formula; the whisper-family table is the reading taken."""
    half = d // 2
    inc = math.log(max_timescale) / (half - 1)
    inv = np.exp(-inc * np.arange(half, dtype=np.float64))
    ang = np.arange(length, dtype=np.float64)[:, None] * inv[None, :]
    return np.concatenate([np.sin(ang), np.cos(ang)], axis=1)


# --------------------------------------------------------------------------
# Token counts and the attention-window partition.
# --------------------------------------------------------------------------

def _conv_len(n: int, k: int = 3, s: int = 2, p: int = 1) -> int:
    return (n + 2 * p - k) // s + 1


def token_count(geom, n_samples: int) -> int:
    """Encoder tokens of one clip of n_samples (> n_fft / 2).

    Mel frames F = floor(n_samples / hop): the centred STFT has 1 + floor(n /
    hop) frames and the trailing one is dropped ([MOSS] gotchas).  Conv2D
    stem: the frames are cut into chunks of chunk_frames, the last chunk
    holding the remaining F mod chunk_frames frames when that is not zero;
    each chunk goes through three k3 s2 p1 convolutions along time ([MOSS]
    Architecture "Conv front-end"; the per-chunk application and the short
    last chunk are the readings of the configured chunk size), so a chunk of
    L frames gives ceil(ceil(ceil(L/2)/2)/2) tokens (13 for 100).  Conv1D
    stem: k3 s1 p1 then k3 s2 p1 ([CW] whisper-small geometry).
    """
    if n_samples <= geom.n_fft // 2:
        raise ValueError("reflect padding needs more than n_fft/2 samples")
    frames = n_samples // geom.hop
    if geom.stem == 0:
        full, rest = divmod(frames, geom.chunk_frames)
        total = 0
        for length in [geom.chunk_frames] * full + ([rest] if rest else []):
            t = length
            for _ in range(3):
                t = _conv_len(t)
            total += t
        return total
    return _conv_len(_conv_len(frames, s=1))


def window_partition(geom, n_samples: int, batch: int) -> np.ndarray:
    """cu_seqlens (int32) of the attention windows of a batch of clips.

    Each clip's tokens are tiled from its first token into windows of
    window_tokens; the last window of a clip is short; windows never cross
    clips.  window_tokens == 0 means one window per clip (full attention).
    [MOSS] Architecture, "Audio encoder": windowed (block-diagonal) attention.
    """
    t = token_count(geom, n_samples)
    w = geom.window_tokens if geom.window_tokens else t
    cu = [0]
    for b in range(batch):
        start = b * t
        pos = 0
        while pos < t:
            step = min(w, t - pos)
            pos += step
            cu.append(start + pos)
    return np.asarray(cu, dtype=np.int32)


# --------------------------------------------------------------------------
# Attention.
# --------------------------------------------------------------------------

def _split_heads(x: np.ndarray, n_heads: int) -> np.ndarray:
    t, d = x.shape
    return x.reshape(t, n_heads, d // n_heads).transpose(1, 0, 2)   # [H, T, dh]


def attention_windows(q, k, v, cu, n_heads: int) -> np.ndarray:
    """Block-diagonal attention: for each window [cu[j], cu[j+1]) and head h,
    softmax(Q K^T / sqrt(dh)) V over that window only.  q, k, v: [T, H*dh].
    [MOSS] Architecture, "Audio encoder": windowed (block-diagonal) attention;
    bidirectional, scale 1/sqrt(head_dim) (reading: the standard scale)."""
    out = np.zeros_like(q)
    for j in range(len(cu) - 1):
        a, b = int(cu[j]), int(cu[j + 1])
        qh, kh, vh = (_split_heads(z[a:b], n_heads) for z in (q, k, v))
        s = qh @ kh.transpose(0, 2, 1) / math.sqrt(qh.shape[-1])
        s = s - s.max(axis=-1, keepdims=True)
        p = np.exp(s)
        p = p / p.sum(axis=-1, keepdims=True)
        out[a:b] = (p @ vh).transpose(1, 0, 2).reshape(b - a, -1)
    return out


def window_mask(cu, t: int) -> np.ndarray:
    """Boolean [T, T]: True where query i and key j share a window."""
    wid = np.zeros(t, dtype=np.int64)
    for j in range(len(cu) - 1):
        wid[int(cu[j]):int(cu[j + 1])] = j
    return wid[:, None] == wid[None, :]


def attention_masked(q, k, v, mask, n_heads: int) -> np.ndarray:
    """Full attention over all T tokens with -inf where ``mask`` is False."""
    qh, kh, vh = (_split_heads(z, n_heads) for z in (q, k, v))
    s = qh @ kh.transpose(0, 2, 1) / math.sqrt(qh.shape[-1])
    s = np.where(mask[None], s, -np.inf)
    s = s - s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=-1, keepdims=True)
    return (p @ vh).transpose(1, 0, 2).reshape(q.shape[0], -1)


# --------------------------------------------------------------------------
# Layers.
# --------------------------------------------------------------------------

def linear(x, w, b=None):
    """y = x W^T + b with W [out, in] (torch Linear layout), in float64."""
    y = np.asarray(x, np.float64) @ as64(w).T
    if b is not None:
        y = y + as64(b)
    return y


def _lin(x, W, name, bias=True):
    return linear(x, W[name + ".w"], W[name + ".b"] if bias else None)


def encoder_layer(x: np.ndarray, W, l: int, geom, cu) -> np.ndarray:
    """One pre-LN block: x + Attn(LN1 x), then + fc2(GELU(fc1(LN2 x))).
    [MOSS] Architecture, "Audio encoder" (32-layer pre-LN, d=1280, 20 heads of
    64, FFN 5120); the FFN activation is GELU (reading: the Whisper/Qwen audio
    tower convention; the pages name no other)."""
    p = f"layers.{l}."
    h = layer_norm(x, as64(W[p + "ln1.g"]), as64(W[p + "ln1.b"]), geom.ln_eps)
    q = _lin(h, W, p + "q")
    k = _lin(h, W, p + "k")
    v = _lin(h, W, p + "v")
    a = attention_windows(q, k, v, cu, geom.n_heads)
    x = x + _lin(a, W, p + "o")
    h = layer_norm(x, as64(W[p + "ln2.g"]), as64(W[p + "ln2.b"]), geom.ln_eps)
    return x + _lin(gelu(_lin(h, W, p + "fc1")), W, p + "fc2")


def stem_conv2d_chunked(mel: np.ndarray, W, geom) -> np.ndarray:
    """Conv2D stem of one clip: mel [M, F] -> tokens [T, d].

    The mel is cut into chunks of chunk_frames frames; each chunk [1, M, 100]
    goes through Conv2D k3 s2 p1 + GELU three times (1 -> C -> C -> C), is
    flattened per time step channel-major (index c * F' + f, F' = M/8), and
    projected by conv_out (no bias); sinusoidal positions 0..12 are added per
    chunk.  [MOSS] Architecture "Conv front-end": 3 x Conv2D stride-2
    (1->480->480->480) -> conv_out (480*16=7680 -> 1280, no bias) ->
    sinusoidal positions.  Readings: GELU after each conv, per-chunk
    application and per-chunk positions (parity unpinned: only trained
    weights could tell these readings apart), channel-major flatten.
    """
    m, f = mel.shape
    cf = geom.chunk_frames
    w1, b1 = as64(W["conv1.w"]), as64(W["conv1.b"])
    w2, b2 = as64(W["conv2.w"]), as64(W["conv2.b"])
    w3, b3 = as64(W["conv3.w"]), as64(W["conv3.b"])
    wo = as64(W["conv_out.w"])
    toks = []
    for c0 in range(0, f, cf):
        x = mel[None, :, c0:c0 + cf]
        x = gelu(conv2d(x, w1, b1))
        x = gelu(conv2d(x, w2, b2))
        x = gelu(conv2d(x, w3, b3))                     # [C, F', T']
        c, fq, tt = x.shape
        flat = x.transpose(2, 0, 1).reshape(tt, c * fq)  # row t: [c * F' + f]
        y = flat @ wo.T
        y = y + sinusoids(tt, geom.d_model)
        toks.append(y)
    return np.concatenate(toks, axis=0)


def stem_conv1d(mel: np.ndarray, W, geom) -> np.ndarray:
    """Whisper stem of one clip: mel [M, F] -> GELU(Conv1D k3 s1 p1) ->
    GELU(Conv1D k3 s2 p1) -> [F/2, d] + global sinusoidal positions.
    [CW] What this exports instead (whisper-small geometry) and Results (1500
    encoder frames for a 30 s window)."""
    x = gelu(conv1d(mel, as64(W["conv1.w"]), as64(W["conv1.b"]), stride=1))
    x = gelu(conv1d(x, as64(W["conv2.w"]), as64(W["conv2.b"]), stride=2))
    y = x.T
    return y + sinusoids(y.shape[0], geom.d_model)


def encode_tokens(x: np.ndarray, W, geom, cu, taps=None) -> np.ndarray:
    """Transformer tower + head + adapter on tokens x [T, d] with the window
    partition ``cu`` (relative to x).  Returns [T, D_out]."""
    for l in range(geom.n_layers):
        x = encoder_layer(x, W, l, geom, cu)
        if taps is not None and l == 0:
            taps["layer0"] = x.copy()
    if taps is not None:
        taps["encoder"] = x.copy()
    h = layer_norm(x, as64(W["ln_post.g"]), as64(W["ln_post.b"]), geom.ln_eps)
    if geom.proj1_out:
        # [MOSS] Architecture, "Encoder head": ln_post -> proj1 -> GELU -> proj2.
        h = _lin(gelu(_lin(h, W, "proj1")), W, "proj2")
    if taps is not None:
        taps["head"] = h.copy()
    if geom.adapter_hidden:
        # [MOSS] Architecture, "Adapter": gated MLP (SwiGLU) 2048 -> 8192 -> 2048,
        # down(SiLU(gate h) * up h); no biases (reading).
        g = h @ as64(W["adapter.gate.w"]).T
        u = h @ as64(W["adapter.up.w"]).T
        h = (silu(g) * u) @ as64(W["adapter.down.w"]).T
    return h


def encode_clip(pcm: np.ndarray, W, geom, taps=None, windows=None) -> np.ndarray:
    """Forward pass of one clip: PCM [n] -> [T, D_out].

    ``windows`` (optional list of window indices of this clip) restricts the
    tower to those windows.  This is exact, not an approximation: windows are
    independent (attention never crosses a window; every other step acts per
    token or per conv chunk), so the rows of a window depend only on the
    chunks of that window and on the clip's mel maximum.  Returns the rows of
    the selected windows, in order.
    """
    mel = log_mel(pcm, geom.n_mels, geom.n_fft, geom.hop)
    if taps is not None:
        taps["mel"] = mel
    n = pcm.shape[0]
    cu = window_partition(geom, n, 1)
    if windows is None:
        sel = list(range(len(cu) - 1))
    else:
        sel = list(windows)
    if geom.stem == 0:
        t_chunk = token_count(geom, geom.chunk_frames * geom.hop)
        parts, cu_sel = [], [0]
        for j in sel:
            a, b = int(cu[j]), int(cu[j + 1])
            c0, c1 = a // t_chunk, -(-b // t_chunk)
            toks = stem_conv2d_chunked(mel[:, c0 * geom.chunk_frames:c1 * geom.chunk_frames], W, geom)
            toks = toks[a - c0 * t_chunk:b - c0 * t_chunk]
            parts.append(toks)
            cu_sel.append(cu_sel[-1] + (b - a))
        x = np.concatenate(parts, axis=0)
        cu_rel = np.asarray(cu_sel, dtype=np.int32)
    else:
        x = stem_conv1d(mel, W, geom)
        if windows is not None:
            parts, cu_sel = [], [0]
            for j in sel:
                a, b = int(cu[j]), int(cu[j + 1])
                parts.append(x[a:b])
                cu_sel.append(cu_sel[-1] + (b - a))
            x = np.concatenate(parts, axis=0)
            cu_rel = np.asarray(cu_sel, dtype=np.int32)
        else:
            cu_rel = cu
    if taps is not None:
        taps["stem"] = x.copy()
    return encode_tokens(x, W, geom, cu_rel, taps)


def encode_stream(pcm: np.ndarray, W, geom) -> np.ndarray:
    """Streaming encoder output of one stream of PCM, [T, D_out].

    The stream is cut into attention windows of window_tokens tokens, i.e.
    window_tokens / (tokens per chunk) conv chunks of mel frames (800 frames,
    8 s, for windows of 104 tokens), and each window is encoded on its own
    ([MOSS] Architecture, "Audio encoder": windowed, block-diagonal attention,
    so windows are independent once their tokens exist).  Reading for live
    input: the frames are the centred STFT frames of the whole stream (the
    stream's own samples on both sides of a window boundary, reflect padding
    only at the stream's start and end), but each window's log-mel is clamped
    and scaled with the maximum over that window's frames, since a live stream
    cannot know the maximum of audio that has not arrived.  The last window
    may be short (a short last chunk, as for any clip).
    """
    t_chunk = token_count(geom, geom.chunk_frames * geom.hop)
    if geom.stem != 0 or not geom.window_tokens or geom.window_tokens % t_chunk:
        raise ValueError("streaming needs the chunked stem and windows of whole chunks")
    wf = geom.window_tokens // t_chunk * geom.chunk_frames
    p = power_spectrum(pcm, geom.n_fft, geom.hop)                 # [F, n_fft/2 + 1], whole stream
    lg = np.log10(np.maximum(p @ mel_filterbank(geom.n_fft // 2 + 1, geom.n_mels), 1e-10))
    outs = []
    for f0 in range(0, lg.shape[0], wf):
        w = lg[f0:f0 + wf]
        w = np.maximum(w, w.max() - 8.0)
        x = stem_conv2d_chunked(((w + 4.0) / 4.0).T, W, geom)
        outs.append(encode_tokens(x, W, geom, np.array([0, x.shape[0]], dtype=np.int32)))
    return np.concatenate(outs, axis=0)


def forward(pcm: np.ndarray, W, geom, taps=None) -> np.ndarray:
    """Batch forward: PCM [B, n] -> [B, T, D_out]; clips are independent
    (per-clip mel maximum, windows never cross clips)."""
    pcm = np.asarray(pcm)
    outs = []
    for b in range(pcm.shape[0]):
        t = {} if taps is not None else None
        outs.append(encode_clip(pcm[b], W, geom, t))
        if taps is not None:
            taps.setdefault("clips", []).append(t)
    return np.stack(outs)


# --------------------------------------------------------------------------
# Audio injection.
# --------------------------------------------------------------------------

def splice_embeddings(ids, placeholder: int, table, frames) -> np.ndarray:
    """LLM input embeddings of a prompt with the audio spliced in, float64
    [len(ids), D]: position i takes the next unused adapter frame when its id
    is the placeholder, else the token's row of the embedding table.
    [MOSS] Architecture, "Audio injection" row (placeholder positions get
    their token embedding replaced by the adapter output frames) and
    "Prompt" row (ChatML framing around the audio).  Raises ValueError when
    the placeholder count differs from the number of frames or an id is not
    a row of the table."""
    ids = [int(i) for i in np.asarray(ids).reshape(-1)]
    table = as64(table)
    frames = as64(frames)
    if sum(1 for i in ids if i == placeholder) != frames.shape[0]:
        raise ValueError("placeholder count differs from the number of frames")
    out = np.zeros((len(ids), table.shape[1]), dtype=np.float64)
    used = 0
    for pos, tok in enumerate(ids):
        if tok == placeholder:
            out[pos] = frames[used]
            used += 1
        else:
            if not 0 <= tok < table.shape[0]:
                raise ValueError(f"token id {tok} is not a row of the table")
            out[pos] = table[tok]
    return out
