"""Python binding of the B200 ASR audio-encoder library (``libasr_enc.so``).

Argument marshalling only: every step of the forward pass runs in the
library's CUDA kernels.  PyTorch supplies device memory (through the
allocator callback and workspace tensors) and streams.  There is no CPU
fallback: importing this package fails loudly when the shared library is
missing, and every call raises on a non-OK status.

The entry points mirror ``include/asr_enc.h`` and ``include/asr_ops.h``:
  tokens, windows, weight_names            geometry queries (host only)
  Encoder(geometry, weights)               asr_enc_create / asr_enc_destroy
  Encoder.forward / forward_host           asr_enc_forward / asr_enc_forward_host
  Encoder.forward_varlen / forward_host_varlen  variable-length batches
  Encoder.sync_status, set_taps, tap       status word and per-stage taps
  log_mel, linear, layer_norm, attention,
  wait_probe                               kernel-level ops
  splice_embeddings                        asr_splice_embeddings / asr_splice_check
  Stream(encoder).push / finish            asr_stream_* (live input, window by window)
"""
from __future__ import annotations

import ctypes
import os

__all__ = ["lib", "LIB_PATH", "AsrError", "Geometry", "tokens", "windows", "weight_names", "Encoder", "Stream",
           "log_mel", "linear", "linear_tf32", "layer_norm", "attention", "gelu", "wait_probe", "splice_embeddings", "TAP_MEL", "TAP_STEM",
           "TAP_LAYER0", "TAP_ENCODER", "TAP_HEAD", "EPI_BF16", "EPI_BF16_GELU", "EPI_F32_RESID",
           "EPI_F32", "EPI_SWIGLU"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libasr_enc.so")

TAP_MEL, TAP_STEM, TAP_LAYER0, TAP_ENCODER, TAP_HEAD = range(5)
EPI_BF16, EPI_BF16_GELU, EPI_F32_RESID, EPI_F32, EPI_SWIGLU = range(5)
STATUS = {0: "ASR_OK", 1: "ASR_E_INVAL", 2: "ASR_E_UNSUPPORTED", 3: "ASR_E_NOMEM", 4: "ASR_E_CUDA",
          5: "ASR_E_WORKSPACE", 6: "ASR_E_DEVICE_TIMEOUT"}


class AsrError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS.get(code, code)}: {msg}")
        self.code = code


class Geometry(ctypes.Structure):
    _fields_ = [("stem", ctypes.c_int), ("n_mels", ctypes.c_int), ("n_fft", ctypes.c_int),
                ("hop", ctypes.c_int), ("chunk_frames", ctypes.c_int), ("conv_ch", ctypes.c_int),
                ("d_model", ctypes.c_int), ("n_heads", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("d_ffn", ctypes.c_int), ("n_layers", ctypes.c_int), ("window_tokens", ctypes.c_int),
                ("pos_mode", ctypes.c_int), ("proj1_out", ctypes.c_int), ("proj2_out", ctypes.c_int),
                ("adapter_hidden", ctypes.c_int), ("adapter_out", ctypes.c_int), ("ln_eps", ctypes.c_float),
                ("dtype", ctypes.c_int)]

    @classmethod
    def of(cls, g) -> "Geometry":
        if isinstance(g, cls):
            return g
        d = g if isinstance(g, dict) else {f: getattr(g, f) for f, _ in cls._fields_}
        return cls(**{f: d[f] for f, _ in cls._fields_})


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python speech_recognition_audio_b200/build.py` "
                          "(there is no CPU fallback)")
    L = ctypes.CDLL(LIB_PATH)
    P, I, I64, SZ, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
    G = ctypes.POINTER(Geometry)
    sig = {
        "asr_enc_weight_count": (I, [G]),
        "asr_enc_weight_info": (I, [G, I, ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(I), ctypes.POINTER(I64)]),
        "asr_enc_tokens": (I64, [G, I64]),
        "asr_enc_windows": (I, [G, I64, I, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(I)]),
        "asr_enc_create": (I, [G, ctypes.POINTER(P), I, P, P, P, P, ctypes.POINTER(P)]),
        "asr_enc_destroy": (None, [P]),
        "asr_enc_workspace_size": (SZ, [P, I64, I]),
        "asr_enc_forward": (I, [P, P, I64, I, P, ctypes.POINTER(I64), P, SZ, P]),
        "asr_enc_forward_host": (I, [P, P, I64, I, P, ctypes.POINTER(I64), P, SZ, P]),
        "asr_enc_workspace_size_varlen": (SZ, [P, ctypes.POINTER(I64), I]),
        "asr_enc_forward_varlen": (I, [P, P, ctypes.POINTER(I64), I, P, ctypes.POINTER(I64), P, SZ, P]),
        "asr_enc_forward_host_varlen": (I, [P, P, ctypes.POINTER(I64), I, P, ctypes.POINTER(I64), P, SZ, P]),
        "asr_enc_sync_status": (I, [P]),
        "asr_enc_set_taps": (I, [P, ctypes.c_uint]),
        "asr_enc_tap": (I, [P, I, P, SZ, P]),
        "asr_enc_last_error": (ctypes.c_char_p, [P]),
        "asr_enc_profile": (I, [P, I]),
        "asr_enc_set_graphs": (I, [P, I]),
        "asr_enc_set_ln_fusion": (I, [P, I]),
        "asr_enc_ln_fusion": (I, [P, ctypes.POINTER(I)]),
        "asr_enc_profile_read": (I, [P, I, ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(ctypes.c_double),
                                     ctypes.POINTER(I)]),
        "asr_enc_last_launches": (I, [P]),
        "asr_op_log_mel_ws_size": (SZ, [I]),
        "asr_op_log_mel": (I, [P, I64, I, I, P, P, SZ, P]),
        "asr_op_log_mel_noalloc": (I, [P, I64, I, I, P, P]),
        "asr_op_linear_ws_size": (SZ, []),
        "asr_op_linear": (I, [P, P, P, I64, I, I, I, I, P, P, SZ, P]),
        "asr_op_linear_tf32": (I, [P, P, P, I64, I, I, I, I, P, P, SZ, P]),
        "asr_op_linear_resid_ln_ws_size": (SZ, [I64, I]),
        "asr_op_linear_resid_ln": (I, [P, P, P, P, P, ctypes.c_float, I64, I, I, P, P, P, SZ, P]),
        "asr_op_layer_norm": (I, [P, P, P, I64, I, F, P, I, P]),
        "asr_op_attention_ws_size": (SZ, []),
        "asr_op_attention": (I, [P, P, I, I, I64, I, P, P, SZ, P]),
        "asr_op_gelu": (I, [P, P, I64, P]),
        "asr_op_wait_probe": (I, [I64, P, P]),
        "asr_stream_window_tokens": (I64, [P]),
        "asr_stream_workspace_size": (SZ, [P, I]),
        "asr_stream_create": (I, [P, ctypes.POINTER(P)]),
        "asr_stream_push": (I, [P, P, I64, P, I64, ctypes.POINTER(I64), P, SZ, P]),
        "asr_stream_finish": (I, [P, P, I64, ctypes.POINTER(I64), P, SZ, P]),
        "asr_stream_destroy": (None, [P]),
        "asr_splice_ws_size": (SZ, [I64]),
        "asr_splice_embeddings": (I, [P, I64, ctypes.c_int32, P, I, I, P, I64, I, P, I, P, SZ, P]),
        "asr_splice_check": (I, [P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


lib = _load()

ALLOC_FN = ctypes.CFUNCTYPE(ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t)
FREE_FN = ctypes.CFUNCTYPE(None, ctypes.c_void_p, ctypes.c_void_p)


def _check(code: int, handle=None):
    if code != 0:
        msg = lib.asr_enc_last_error(handle)
        raise AsrError(code, msg.decode() if msg else "")


def _stream(stream):
    import torch
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def tokens(geometry, n_samples: int) -> int:
    """Tokens per clip (bit-exact host query); -1 for unsupported sizes."""
    g = Geometry.of(geometry)
    return int(lib.asr_enc_tokens(ctypes.byref(g), int(n_samples)))


def windows(geometry, n_samples: int, batch: int):
    """Attention-window cumulative offsets (list of int) of a batch."""
    g = Geometry.of(geometry)
    n = ctypes.c_int(0)
    _check(lib.asr_enc_windows(ctypes.byref(g), int(n_samples), int(batch), None, ctypes.byref(n)))
    cu = (ctypes.c_int32 * (n.value + 1))()
    cap = ctypes.c_int(n.value + 1)
    _check(lib.asr_enc_windows(ctypes.byref(g), int(n_samples), int(batch), cu, ctypes.byref(cap)))
    return list(cu)


def weight_names(geometry):
    """[(name, shape)] in the order asr_enc_create expects."""
    g = Geometry.of(geometry)
    count = lib.asr_enc_weight_count(ctypes.byref(g))
    if count < 0:
        raise AsrError(1, "invalid geometry")
    out = []
    for i in range(count):
        name = ctypes.c_char_p()
        nd = ctypes.c_int()
        shape = (ctypes.c_int64 * 4)()
        _check(lib.asr_enc_weight_info(ctypes.byref(g), i, ctypes.byref(name), ctypes.byref(nd), shape))
        out.append((name.value.decode(), tuple(shape[k] for k in range(nd.value))))
    return out


class _TorchAllocator:
    """Device memory for the library, from torch's caching allocator."""

    def __init__(self, device):
        self.device = device
        self.keep = {}
        self.alloc_cb = ALLOC_FN(self._alloc)
        self.free_cb = FREE_FN(self._free)

    def _alloc(self, ctx, nbytes):
        import torch
        try:
            t = torch.empty(int(nbytes), dtype=torch.uint8, device=self.device)
        except Exception:  # out of memory -> NULL -> ASR_E_NOMEM
            return None
        self.keep[t.data_ptr()] = t
        return t.data_ptr()

    def _free(self, ctx, ptr):
        self.keep.pop(ptr, None)


class Encoder:
    """One encoder instance: weights repacked on the device by asr_enc_create.

    ``weights``: mapping name -> CUDA tensor (geometry dtype), names and shapes
    as listed by ``weight_names``.
    """

    def __init__(self, geometry, weights, stream=None):
        import torch
        self.geometry = Geometry.of(geometry)
        specs = weight_names(self.geometry)
        ptrs = (ctypes.c_void_p * len(specs))()
        for i, (name, shape) in enumerate(specs):
            t = weights[name]
            if not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != tuple(shape):
                raise ValueError(f"weight {name}: need a contiguous CUDA tensor of shape {shape}")
            ptrs[i] = t.data_ptr()
        self.device = torch.cuda.current_device()
        self._alloc = _TorchAllocator(torch.device("cuda", self.device))
        h = ctypes.c_void_p()
        _check(lib.asr_enc_create(ctypes.byref(self.geometry), ptrs, len(specs),
                                  ctypes.cast(self._alloc.alloc_cb, ctypes.c_void_p),
                                  ctypes.cast(self._alloc.free_cb, ctypes.c_void_p), None, _stream(stream),
                                  ctypes.byref(h)))
        self.handle = h
        self._ws = None
        self.taps = 0

    def close(self):
        if getattr(self, "handle", None):
            lib.asr_enc_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def d_out(self) -> int:
        g = self.geometry
        return g.adapter_out if g.adapter_hidden else (g.proj2_out if g.proj2_out else g.d_model)

    def tokens(self, n_samples: int) -> int:
        return tokens(self.geometry, n_samples)

    def workspace_size(self, n_samples: int, batch: int) -> int:
        return int(lib.asr_enc_workspace_size(self.handle, int(n_samples), int(batch)))

    def workspace(self, n_samples: int, batch: int):
        """A cached workspace tensor big enough for (n_samples, batch)."""
        import torch
        need = self.workspace_size(n_samples, batch)
        if need == 0:
            raise AsrError(1, lib.asr_enc_last_error(self.handle).decode() or "unsupported size")
        if self._ws is None or self._ws.numel() < need:
            self._ws = None
            self._ws = torch.empty(need, dtype=torch.uint8, device=torch.device("cuda", self.device))
        return self._ws

    def forward(self, pcm, out=None, workspace=None, stream=None):
        """pcm: CUDA float32 [B, n] -> CUDA float32 [B, T, D_out] (asynchronous)."""
        import torch
        if pcm.dtype != torch.float32 or not pcm.is_cuda or pcm.dim() != 2 or not pcm.is_contiguous():
            raise ValueError("pcm must be a contiguous CUDA float32 tensor [batch, n_samples]")
        B, n = pcm.shape
        T = self.tokens(n)
        if T <= 0:
            raise AsrError(2, f"n_samples={n} is not supported by this geometry")
        if out is None:
            out = torch.empty((B, T, self.d_out), dtype=torch.float32, device=pcm.device)
        ws = workspace if workspace is not None else self.workspace(n, B)
        nt = ctypes.c_int64()
        _check(lib.asr_enc_forward(self.handle, _ptr(pcm), n, B, _ptr(out), ctypes.byref(nt), _ptr(ws),
                                   ws.numel() * ws.element_size(), _stream(stream)), self.handle)
        return out

    def forward_host(self, pcm_host, out_host=None, workspace=None, stream=None):
        """Host float32 [B, n] (pinned for speed) -> host float32 [B, T, D_out]; synchronous."""
        import torch
        if pcm_host.dtype != torch.float32 or pcm_host.is_cuda or pcm_host.dim() != 2 or not pcm_host.is_contiguous():
            raise ValueError("pcm_host must be a contiguous CPU float32 tensor [batch, n_samples]")
        B, n = pcm_host.shape
        T = self.tokens(n)
        if out_host is None:
            out_host = torch.empty((B, T, self.d_out), dtype=torch.float32, pin_memory=pcm_host.is_pinned())
        ws = workspace if workspace is not None else self.workspace(n, B)
        nt = ctypes.c_int64()
        _check(lib.asr_enc_forward_host(self.handle, _ptr(pcm_host), n, B, _ptr(out_host), ctypes.byref(nt),
                                        _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)), self.handle)
        return out_host

    def _ws_varlen(self, ns, workspace):
        import torch
        arr = (ctypes.c_int64 * len(ns))(*[int(v) for v in ns])
        need = int(lib.asr_enc_workspace_size_varlen(self.handle, arr, len(ns)))
        if need == 0:
            raise AsrError(2, "unsupported variable-length batch")
        if workspace is not None:
            return arr, workspace
        if self._ws is None or self._ws.numel() < need:
            self._ws = None
            self._ws = torch.empty(need, dtype=torch.uint8, device=torch.device("cuda", self.device))
        return arr, self._ws

    def forward_varlen(self, pcm, n_samples, out=None, workspace=None, stream=None):
        """Variable-length batch: pcm CUDA float32 [sum n_b] (clips packed),
        n_samples list of per-clip lengths -> (CUDA float32 [sum T_b, D_out],
        list of T_b)."""
        import torch
        if pcm.dtype != torch.float32 or not pcm.is_cuda or pcm.dim() != 1 or not pcm.is_contiguous():
            raise ValueError("pcm must be a contiguous 1-D CUDA float32 tensor (clips packed)")
        if pcm.numel() != sum(int(v) for v in n_samples):
            raise ValueError("pcm length must equal sum(n_samples)")
        toks = [self.tokens(v) for v in n_samples]
        if min(toks) <= 0:
            raise AsrError(2, "a clip length is not supported by this geometry")
        if out is None:
            out = torch.empty((sum(toks), self.d_out), dtype=torch.float32, device=pcm.device)
        arr, ws = self._ws_varlen(n_samples, workspace)
        nt = (ctypes.c_int64 * len(n_samples))()
        _check(lib.asr_enc_forward_varlen(self.handle, _ptr(pcm), arr, len(n_samples), _ptr(out), nt, _ptr(ws),
                                          ws.numel() * ws.element_size(), _stream(stream)), self.handle)
        return out, list(nt)

    def forward_host_varlen(self, pcm_host, n_samples, out_host=None, workspace=None, stream=None):
        """Host form of forward_varlen (synchronous)."""
        import torch
        toks = [self.tokens(v) for v in n_samples]
        if out_host is None:
            out_host = torch.empty((sum(toks), self.d_out), dtype=torch.float32, pin_memory=pcm_host.is_pinned())
        arr, ws = self._ws_varlen(n_samples, workspace)
        nt = (ctypes.c_int64 * len(n_samples))()
        _check(lib.asr_enc_forward_host_varlen(self.handle, _ptr(pcm_host), arr, len(n_samples), _ptr(out_host), nt,
                                               _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)), self.handle)
        return out_host, list(nt)

    def sync_status(self):
        _check(lib.asr_enc_sync_status(self.handle), self.handle)

    def set_graphs(self, enable: bool):
        """Record uniform forwards as CUDA graphs and replay them (default on)."""
        _check(lib.asr_enc_set_graphs(self.handle, 1 if enable else 0), self.handle)

    def set_ln_fusion(self, enable: bool):
        """Next-block LayerNorm computed in fc2's epilogue (default off; see asr_enc.h)."""
        _check(lib.asr_enc_set_ln_fusion(self.handle, 1 if enable else 0), self.handle)

    def ln_fusion(self) -> bool:
        """Whether forwards compute the LayerNorms in the residual GEMMs' epilogues."""
        v = ctypes.c_int(0)
        _check(lib.asr_enc_ln_fusion(self.handle, ctypes.byref(v)), self.handle)
        return bool(v.value)

    def set_taps(self, mask: int):
        _check(lib.asr_enc_set_taps(self.handle, int(mask)), self.handle)
        self.taps = int(mask)
        self._ws = None

    def tap(self, stage: int, shape, stream=None):
        import torch
        dst = torch.empty(shape, dtype=torch.float32, device=torch.device("cuda", self.device))
        _check(lib.asr_enc_tap(self.handle, int(stage), _ptr(dst), dst.numel() * 4, _stream(stream)), self.handle)
        return dst


# ------------------------------------------------------------------ ops

def log_mel(pcm, n_mels: int, stream=None):
    """pcm CUDA float32 [B, n] -> normalised log-mel CUDA float32 [B, n_mels, n/160]."""
    import torch
    B, n = pcm.shape
    mel = torch.empty((B, n_mels, n // 160), dtype=torch.float32, device=pcm.device)
    ws = torch.empty(int(lib.asr_op_log_mel_ws_size(B)), dtype=torch.uint8, device=pcm.device)
    _check(lib.asr_op_log_mel(_ptr(pcm), n, B, n_mels, _ptr(mel), _ptr(ws), ws.numel(), _stream(stream)))
    return mel


def linear(x, w, bias=None, epi: int = EPI_BF16, out=None, tile_n: int = 0, stream=None):
    """x bf16 [M, K], w bf16 [N, K], bias f32 [N] -> epilogue(x w^T + bias) (see asr_ops.h)."""
    import torch
    M, K = x.shape
    N = w.shape[0]
    if out is None:
        if epi in (EPI_BF16, EPI_BF16_GELU):
            out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
        elif epi == EPI_SWIGLU:
            out = torch.empty((M, N // 2), dtype=torch.bfloat16, device=x.device)
        elif epi == EPI_F32:
            out = torch.empty((M, N), dtype=torch.float32, device=x.device)
        else:
            raise ValueError("EPI_F32_RESID needs `out` (updated in place)")
    ws = torch.empty(int(lib.asr_op_linear_ws_size()), dtype=torch.uint8, device=x.device)
    _check(lib.asr_op_linear(_ptr(x), _ptr(w), _ptr(bias), M, N, K, epi, int(tile_n), _ptr(out), _ptr(ws),
                             ws.numel(), _stream(stream)))
    return out


def linear_resid_ln(x, w, bias, gamma, beta, y, eps: float = 1e-5, h=None, stream=None):
    """y f32 [M, N] += x w^T + bias (in place), then h bf16 [M, N] = LayerNorm(y) * gamma + beta, in one
    launch (asr_op_linear_resid_ln).  Returns h."""
    import torch
    M, K = x.shape
    N = w.shape[0]
    if h is None:
        h = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    ws = torch.empty(int(lib.asr_op_linear_resid_ln_ws_size(M, N)), dtype=torch.uint8, device=x.device)
    _check(lib.asr_op_linear_resid_ln(_ptr(x), _ptr(w), _ptr(bias), _ptr(gamma), _ptr(beta), float(eps), M, N, K,
                                      _ptr(y), _ptr(h), _ptr(ws), ws.numel(), _stream(stream)))
    return h


def linear_tf32(x, w, bias=None, epi: int = EPI_F32, out=None, tile_n: int = 0, stream=None):
    """x float32 [M, K], w float32 [N, K] -> epilogue(x w^T + bias) in fp32,
    multiplied on the tensor cores as tf32 (asr_op_linear_tf32)."""
    import torch
    M, K = x.shape
    N = w.shape[0]
    if out is None:
        if epi == EPI_F32_RESID:
            raise ValueError("EPI_F32_RESID needs `out` (updated in place)")
        out = torch.empty((M, N // 2 if epi == EPI_SWIGLU else N), dtype=torch.float32, device=x.device)
    ws = torch.empty(256, dtype=torch.uint8, device=x.device)
    _check(lib.asr_op_linear_tf32(_ptr(x), _ptr(w), _ptr(bias), M, N, K, epi, int(tile_n), _ptr(out), _ptr(ws),
                                  ws.numel(), _stream(stream)))
    return out


def layer_norm(x, g, b, eps: float = 1e-5, out_f32: bool = False, stream=None):
    import torch
    M, D = x.shape
    y = torch.empty((M, D), dtype=torch.float32 if out_f32 else torch.bfloat16, device=x.device)
    _check(lib.asr_op_layer_norm(_ptr(x), _ptr(g), _ptr(b), M, D, eps, _ptr(y), int(out_f32), _stream(stream)))
    return y


def attention(qkv, cu, n_heads: int, stream=None):
    """qkv bf16 [T, 3*H*64], cu int32 CUDA [n_seg+1] -> bf16 [T, H*64]."""
    import torch
    T = qkv.shape[0]
    cu_host = cu.cpu().tolist()
    max_seg = max(b - a for a, b in zip(cu_host[:-1], cu_host[1:]))
    out = torch.empty((T, n_heads * 64), dtype=torch.bfloat16, device=qkv.device)
    ws = torch.zeros(int(lib.asr_op_attention_ws_size()), dtype=torch.uint8, device=qkv.device)
    _check(lib.asr_op_attention(_ptr(qkv), _ptr(cu), len(cu_host) - 1, max_seg, T, n_heads, _ptr(out), _ptr(ws),
                                ws.numel(), _stream(stream)))
    if int(ws[:4].view(torch.int32).item()) != 0:
        raise AsrError(6, "attention: a bounded device wait gave up")
    return out


def gelu(x, stream=None):
    """The device GELU: x CUDA float32 -> float32 of the same shape."""
    import torch
    y = torch.empty_like(x)
    _check(lib.asr_op_gelu(_ptr(x), _ptr(y), x.numel(), _stream(stream)))
    return y


def wait_probe(limit_ns: int, stream=None) -> int:
    """Run the bounded-wait self-check; returns the status word it wrote."""
    import torch
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    _check(lib.asr_op_wait_probe(int(limit_ns), _ptr(st), _stream(stream)))
    torch.cuda.synchronize()
    return int(st.item())


_DTYPE_CODE = {"bfloat16": 0, "float32": 1, "float16": 2}


def splice_embeddings(ids, placeholder: int, table, frames, out_dtype=None, stream=None, check: bool = True):
    """LLM input embeddings with the audio spliced in: ids CUDA int32 [n],
    table CUDA [vocab, D] (bf16 / f16 / f32), frames CUDA float32 [n_frames, D]
    -> CUDA [n, D] of out_dtype (default: the table's dtype).  With check the
    call synchronises and raises on a bad id or a placeholder/frame count
    mismatch."""
    import torch
    out_dtype = out_dtype or table.dtype
    n = ids.numel()
    D = table.shape[1]
    out = torch.empty((n, D), dtype=out_dtype, device=ids.device)
    ws = torch.empty(int(lib.asr_splice_ws_size(n)), dtype=torch.uint8, device=ids.device)
    code = lambda t: _DTYPE_CODE[str(t).replace("torch.", "")]
    st = _stream(stream)
    _check(lib.asr_splice_embeddings(_ptr(ids), n, int(placeholder), _ptr(table), table.shape[0], code(table.dtype),
                                     _ptr(frames), frames.shape[0] if frames is not None else 0, D, _ptr(out),
                                     code(out_dtype), _ptr(ws), ws.numel(), st))
    if check:
        _check(lib.asr_splice_check(_ptr(ws), st))
    return out


class Stream:
    """Live input on an Encoder: push() device float32 samples as they arrive;
    each call returns the rows of the attention windows that became ready
    (CUDA float32 [rows, D_out]); finish() returns the rows of the last,
    possibly short, window.  See asr_enc.h, streaming."""

    def __init__(self, encoder, stream=None):
        self.enc = encoder
        self.wtok = int(lib.asr_stream_window_tokens(encoder.handle))
        if self.wtok <= 0:
            raise AsrError(2, "streaming needs the chunked conv2d stem and windows of whole chunks")
        g = encoder.geometry
        self.win_samples = self.wtok // 13 * g.chunk_frames * g.hop
        self.half, self.hop = g.n_fft // 2, g.hop
        h = ctypes.c_void_p()
        _check(lib.asr_stream_create(encoder.handle, ctypes.byref(h)), encoder.handle)
        self.handle = h
        self.total = 0
        self.done = 0
        self.stream = stream
        self._ws = None

    def _ws_for(self, windows):
        import torch
        need = int(lib.asr_stream_workspace_size(self.enc.handle, max(windows, 1)))
        if self._ws is None or self._ws.numel() < need:
            self._ws = None
            self._ws = torch.empty(need, dtype=torch.uint8, device=torch.device("cuda", self.enc.device))
        return self._ws

    def _ready(self, total):
        k = 0
        while (self.done + k + 1) * self.win_samples - self.hop + self.half <= total:
            k += 1
        return k

    def push(self, pcm):
        import torch
        if pcm.dtype != torch.float32 or not pcm.is_cuda or pcm.dim() != 1 or not pcm.is_contiguous():
            raise ValueError("pcm must be a contiguous 1-D CUDA float32 tensor")
        k = self._ready(self.total + pcm.numel())
        out = torch.empty((max(k, 1) * self.wtok, self.enc.d_out), dtype=torch.float32, device=pcm.device)
        ws = self._ws_for(k)
        rows = ctypes.c_int64()
        _check(lib.asr_stream_push(self.handle, _ptr(pcm), pcm.numel(), _ptr(out), out.shape[0], ctypes.byref(rows),
                                   _ptr(ws), ws.numel(), _stream(self.stream)), self.enc.handle)
        self.total += pcm.numel()
        self.done += k
        return out[: rows.value]

    def finish(self):
        import torch
        out = torch.empty((self.wtok, self.enc.d_out), dtype=torch.float32, device=torch.device("cuda", self.enc.device))
        ws = self._ws_for(1)
        rows = ctypes.c_int64()
        _check(lib.asr_stream_finish(self.handle, _ptr(out), out.shape[0], ctypes.byref(rows), _ptr(ws), ws.numel(),
                                     _stream(self.stream)), self.enc.handle)
        return out[: rows.value]

    def close(self):
        if getattr(self, "handle", None):
            lib.asr_stream_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
