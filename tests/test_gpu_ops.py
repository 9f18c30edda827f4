"""Kernel-level parity of the CUDA library against the oracle (GPU).

Each op is called through the C ABI (include/asr_ops.h) on seeded inputs and
compared element by element with the oracle's float64 definition of the same
step, at sizes that span several tiles and a ragged tail.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

sra = pytest.importorskip("speech_recognition_audio_b200")


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


# ------------------------------------------------------------------ GEMM
@pytest.mark.parametrize("M,N,K", [(1, 256, 64), (13, 64, 576), (100, 128, 72), (300, 512, 1280),
                                   (1000, 1280, 1280), (777, 480, 4320), (6240, 3840, 1280),
                                   (200, 768, 2304), (129, 2048, 8192)])
def test_linear_bf16_bias(M, N, K):
    rng = np.random.default_rng(M * 7 + N + K)
    x = _bf16(rng.normal(size=(M, K)))
    w = _bf16(rng.normal(size=(N, K)) * 0.05)
    b = torch.from_numpy(rng.normal(size=N).astype(np.float32))
    y = sra.linear(x.cuda(), w.cuda(), b.cuda(), sra.EPI_BF16)
    torch.cuda.synchronize()
    ref = oracle.linear(x.float().numpy(), w, b.numpy())
    got = y.float().cpu().numpy()
    err = np.abs(got - ref)
    tol = 2.0 ** -8 * np.abs(ref) + 1e-3 * np.sqrt(K / 64) * 0.05
    assert (err <= tol).all(), f"max err {err.max()} (M={M} N={N} K={K})"


@pytest.mark.parametrize("tile_n", [256, 160, 128, 64, -256, -128])
@pytest.mark.parametrize("M,N,K", [(6240, 1280, 1280), (300, 480, 4320), (257, 2560, 96), (20000, 480, 16)])
def test_linear_tile_modes(tile_n, M, N, K):
    """Every tile shape of the engine (one SM 128 x tile_n, or a CTA pair
    256 x -tile_n) gives the same result, including ragged M and N tails
    and a single partial k-block (K = 16, as in conv1)."""
    if tile_n == 160 and N % 160:
        pytest.skip("160-wide tiles need N % 160 == 0")
    rng = np.random.default_rng(M + N + K + tile_n)
    x = _bf16(rng.normal(size=(M, K)))
    w = _bf16(rng.normal(size=(N, K)) * 0.05)
    b = torch.from_numpy(rng.normal(size=N).astype(np.float32))
    r0 = rng.normal(size=(M, N)).astype(np.float32)
    out = torch.from_numpy(r0).cuda()
    sra.linear(x.cuda(), w.cuda(), b.cuda(), sra.EPI_F32_RESID, out=out, tile_n=tile_n)
    ref = r0 + oracle.linear(x.float().numpy(), w, b.numpy())
    np.testing.assert_allclose(out.cpu().numpy(), ref, rtol=1e-4, atol=2e-4 * np.sqrt(K / 64))
    y = sra.linear(x.cuda(), w.cuda(), b.cuda(), sra.EPI_BF16_GELU, tile_n=tile_n).float().cpu().numpy()
    g = oracle.gelu(ref - r0)
    assert np.abs(y - g).max() <= 2.0 ** -8 * np.abs(g).max() + 1e-3


@pytest.mark.parametrize("M,N,K,epi", [(6240, 1280, 5120, "resid"), (6240, 1280, 2560, "resid"),
                                       (3000, 2048, 4096, "resid"), (600, 1280, 5120, "resid"),
                                       (3000, 2048, 4096, "f32")])
def test_linear_stream_k(M, N, K, epi):
    """The residual epilogue on CTA-pair tiles runs stream-K when the tile
    count leaves a ragged last wave: parity with the oracle, and two runs
    agree bit for bit (a split tile's two updates land in a fixed order)."""
    rng = np.random.default_rng(M + N + K)
    x = _bf16(rng.normal(size=(M, K)))
    w = _bf16(rng.normal(size=(N, K)) * 0.03)
    b = torch.from_numpy(rng.normal(size=N).astype(np.float32))
    acc = oracle.linear(x.float().numpy(), w, b.numpy())
    xc, wc, bc = x.cuda(), w.cuda(), b.cuda()
    runs = []
    for _ in range(2):
        if epi == "resid":
            r0 = np.random.default_rng(5).normal(size=(M, N)).astype(np.float32)
            out = torch.from_numpy(r0).cuda()
            sra.linear(xc, wc, bc, sra.EPI_F32_RESID, out=out, tile_n=-256)
            ref = r0 + acc
        else:
            out = sra.linear(xc, wc, bc, sra.EPI_F32, tile_n=-256)
            ref = acc
        runs.append(out.cpu().numpy())
    np.testing.assert_allclose(runs[0], ref, rtol=1e-4, atol=2e-4 * np.sqrt(K / 64) * 0.6)
    assert np.array_equal(runs[0], runs[1])


@pytest.mark.parametrize("M,N,K,shift", [(6240, 1280, 1280, 0.0), (6240, 1280, 5120, 0.0), (333, 768, 3072, 0.0),
                                         (1, 256, 128, 0.0), (300, 1280, 256, 50.0), (77, 32, 128, 0.0),
                                         (500, 96, 256, -3.0), (1000, 1312, 128, 0.0), (48000, 768, 128, 0.0)])
def test_linear_resid_ln(M, N, K, shift):
    """Residual GEMM + LayerNorm of the updated rows in one launch: y against
    the oracle's r0 + x w^T + b (and bit for bit against the plain residual
    epilogue where that runs whole tiles, K < 40 k-blocks), h against the
    oracle's LayerNorm of it.  Ragged M (partial 32-row groups and 256-row
    tiles), N with a partial last n-tile (96, 1312: halves of warps with 32 or
    no valid columns), a single row, rows with a large common offset (the
    statistics' cancellation), and 188 row blocks (more tiles than pairs)."""
    rng = np.random.default_rng(M + 3 * N + K)
    x = _bf16(rng.normal(size=(M, K)))
    w = _bf16(rng.normal(size=(N, K)) * 0.04)
    b = torch.from_numpy(rng.normal(size=N).astype(np.float32) * 0.1)
    g = torch.from_numpy((1 + 0.1 * rng.normal(size=N)).astype(np.float32))
    be = torch.from_numpy((0.05 * rng.normal(size=N)).astype(np.float32))
    r0 = (rng.normal(size=(M, N)) + shift).astype(np.float32)
    xc, wc, bc = x.cuda(), w.cuda(), b.cuda()
    y = torch.from_numpy(r0).cuda()
    h = sra.linear_resid_ln(xc, wc, bc, g.cuda(), be.cuda(), y, eps=1e-5)
    y2 = torch.from_numpy(r0).cuda()
    h2 = sra.linear_resid_ln(xc, wc, bc, g.cuda(), be.cuda(), y2, eps=1e-5)
    torch.cuda.synchronize()
    yr = r0.astype(np.float64) + oracle.linear(x.float().numpy(), w, b.numpy())
    hr = oracle.layer_norm(yr, g.numpy(), be.numpy(), 1e-5)
    got_y, got_h = y.cpu().numpy(), h.float().cpu().numpy()
    np.testing.assert_allclose(got_y, yr, rtol=1e-5, atol=2e-4 * np.sqrt(K / 64) * 0.8)
    err = np.abs(got_h - hr)
    tol = 2.0 ** -8 * np.abs(hr) + 2e-3
    assert (err <= tol).all(), f"h max err {err.max()} at {np.unravel_index(err.argmax(), err.shape)}"
    assert np.array_equal(got_y, y2.cpu().numpy()) and np.array_equal(got_h, h2.float().cpu().numpy())
    if K < 40 * 64:
        y3 = torch.from_numpy(r0).cuda()
        sra.linear(xc, wc, bc, sra.EPI_F32_RESID, out=y3, tile_n=-256)
        assert np.array_equal(got_y, y3.cpu().numpy())


def test_linear_resid_ln_rejects_unsupported_shapes():
    x = torch.zeros((64, 96), dtype=torch.bfloat16, device="cuda")       # K % 128 != 0
    w = torch.zeros((256, 96), dtype=torch.bfloat16, device="cuda")
    v = torch.zeros(256, device="cuda")
    y = torch.zeros((64, 256), device="cuda")
    with pytest.raises(sra.AsrError):
        sra.linear_resid_ln(x, w, v, v, v, y)
    x = torch.zeros((64, 128), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((48, 128), dtype=torch.bfloat16, device="cuda")      # N % 32 != 0
    with pytest.raises(sra.AsrError):
        sra.linear_resid_ln(x, w, v[:48], v[:48], v[:48], y[:, :48].contiguous())


@pytest.mark.parametrize("epi", ["gelu", "f32", "resid", "swiglu"])
def test_linear_epilogues(epi):
    M, N, K = 333, 1024, 768
    rng = np.random.default_rng(11)
    x = _bf16(rng.normal(size=(M, K)))
    w = _bf16(rng.normal(size=(N, K)) * 0.04)
    b = torch.from_numpy(rng.normal(size=N).astype(np.float32) * 0.1)
    acc = oracle.linear(x.float().numpy(), w, b.numpy())
    if epi == "gelu":
        got = sra.linear(x.cuda(), w.cuda(), b.cuda(), sra.EPI_BF16_GELU).float().cpu().numpy()
        ref = oracle.gelu(acc)
        assert np.abs(got - ref).max() <= 2.0 ** -8 * np.abs(ref).max() + 1e-3
    elif epi == "f32":
        got = sra.linear(x.cuda(), w.cuda(), b.cuda(), sra.EPI_F32).cpu().numpy()
        np.testing.assert_allclose(got, acc, rtol=1e-4, atol=1e-4)
    elif epi == "resid":
        r0 = rng.normal(size=(M, N)).astype(np.float32)
        out = torch.from_numpy(r0).cuda()
        sra.linear(x.cuda(), w.cuda(), b.cuda(), sra.EPI_F32_RESID, out=out)
        np.testing.assert_allclose(out.cpu().numpy(), r0 + acc, rtol=1e-4, atol=1e-4)
    else:
        # rows interleaved in blocks of 16: gate block j then up block j
        wg, wu = w[: N // 2], w[N // 2:]
        wi = torch.stack([wg.view(-1, 16, K), wu.view(-1, 16, K)], 1).reshape(N, K).contiguous()
        got = sra.linear(x.cuda(), wi.cuda(), None, sra.EPI_SWIGLU).float().cpu().numpy()
        xf = x.float().numpy()
        ref = oracle.silu(oracle.linear(xf, wg)) * oracle.linear(xf, wu)
        assert got.shape == (M, N // 2)
        assert np.abs(got - ref).max() <= 2.0 ** -8 * np.abs(ref).max() + 2e-3


@pytest.mark.parametrize("M,N,K,tile_n", [(13, 256, 256, 0), (300, 1024, 1024, 0), (777, 480, 4320, 128),
                                           (129, 512, 64, 64), (1000, 1280, 1280, 256)])
def test_linear_tf32_matches_oracle(M, N, K, tile_n):
    """fp32 operands on kind::tf32: every product sees each operand rounded
    to tf32 (10 explicit mantissa bits), so |error| <= 2^-9 sum |x| |w| plus
    fp32 accumulation."""
    rng = np.random.default_rng(M + N + K)
    x = rng.normal(size=(M, K)).astype(np.float32)
    w = (rng.normal(size=(N, K)) * 0.05).astype(np.float32)
    b = rng.normal(size=N).astype(np.float32)
    xt, wt, bt = (torch.from_numpy(a).cuda() for a in (x, w, b))
    bound = 2.0 ** -9 * (np.abs(x.astype(np.float64)) @ np.abs(w.astype(np.float64)).T) + 1e-5
    ref = oracle.linear(x, w, b)
    y = sra.linear_tf32(xt, wt, bt, sra.EPI_F32, tile_n=tile_n).cpu().numpy()
    assert (np.abs(y - ref) <= bound).all(), np.abs(y - ref).max()
    r0 = rng.normal(size=(M, N)).astype(np.float32)
    out = torch.from_numpy(r0).cuda()
    sra.linear_tf32(xt, wt, bt, sra.EPI_F32_RESID, out=out, tile_n=tile_n)
    assert (np.abs(out.cpu().numpy() - (r0 + ref)) <= bound + 1e-5).all()
    g = sra.linear_tf32(xt, wt, bt, sra.EPI_BF16_GELU, tile_n=tile_n).cpu().numpy()
    # |GELU'| <= 1.13, plus the device GELU's own error (tanh form)
    assert (np.abs(g - oracle.gelu(ref)) <= 1.13 * bound + 4.8e-4 + 2.6e-4 * np.abs(ref)).all()


def test_linear_tf32_swiglu():
    M, N, K = 333, 1024, 768
    rng = np.random.default_rng(12)
    x = rng.normal(size=(M, K)).astype(np.float32)
    w = (rng.normal(size=(N, K)) * 0.04).astype(np.float32)
    wg, wu = w[: N // 2], w[N // 2:]
    wi = np.stack([wg.reshape(-1, 16, K), wu.reshape(-1, 16, K)], 1).reshape(N, K)
    got = sra.linear_tf32(torch.from_numpy(x).cuda(), torch.from_numpy(np.ascontiguousarray(wi)).cuda(), None,
                          sra.EPI_SWIGLU).cpu().numpy()
    ref = oracle.silu(oracle.linear(x, wg)) * oracle.linear(x, wu)
    assert got.shape == (M, N // 2)
    assert np.abs(got - ref).max() <= 2e-3 * max(1.0, np.abs(ref).max())


# ------------------------------------------------------------------ mel
@pytest.mark.parametrize("n_mels,secs,batch,speech", [(128, 1, 1, False), (128, 3, 2, False),
                                                      (80, 2, 3, False), (128, 20, 1, True)])
def test_log_mel(n_mels, secs, batch, speech):
    pcm = np.stack([synth.pcm_clip(16000 * secs, 100 + b, speech) for b in range(batch)])
    got = sra.log_mel(torch.from_numpy(pcm).cuda(), n_mels).cpu().numpy()
    for b in range(batch):
        ref = oracle.log_mel(pcm[b], n_mels)
        assert np.abs(got[b] - ref).max() <= 1e-3


def test_log_mel_ragged_frames():
    # n/160 not a multiple of the kernel's frame group
    pcm = synth.pcm_clip(160 * 123, 7)[None]
    got = sra.log_mel(torch.from_numpy(pcm).cuda(), 128).cpu().numpy()[0]
    ref = oracle.log_mel(pcm[0], 128)
    assert got.shape == ref.shape == (128, 123)
    assert np.abs(got - ref).max() <= 1e-3


# ------------------------------------------------------------------ LN
@pytest.mark.parametrize("M,D", [(1, 256), (77, 768), (6240, 1280), (5, 2048), (48000, 768), (20000, 1280)])
def test_layer_norm(M, D):
    rng = np.random.default_rng(D + M)
    x = (rng.normal(size=(M, D)) * 3 + 0.5).astype(np.float32)
    g = (1 + 0.1 * rng.normal(size=D)).astype(np.float32)
    b = (0.02 * rng.normal(size=D)).astype(np.float32)
    ref = oracle.layer_norm(x.astype(np.float64), g, b, 1e-5)
    y16 = sra.layer_norm(torch.from_numpy(x).cuda(), torch.from_numpy(g).cuda(), torch.from_numpy(b).cuda())
    y32 = sra.layer_norm(torch.from_numpy(x).cuda(), torch.from_numpy(g).cuda(), torch.from_numpy(b).cuda(),
                         out_f32=True)
    np.testing.assert_allclose(y32.cpu().numpy(), ref, rtol=1e-4, atol=1e-4)
    assert np.abs(y16.float().cpu().numpy() - ref).max() <= 2.0 ** -8 * np.abs(ref).max()


def test_layer_norm_forms_agree():
    """Row counts that fit the SMs at once run the single-wave form (rows
    staged in shared memory), larger ones the register form with prefetch:
    the same arithmetic in the same order, so a row normalises to the same
    bits in both."""
    rng = np.random.default_rng(4)
    D = 1280
    big = torch.from_numpy((rng.normal(size=(40000, D)) * 2 + 0.3).astype(np.float32)).cuda()
    g = torch.from_numpy((1 + 0.1 * rng.normal(size=D)).astype(np.float32)).cuda()
    b = torch.from_numpy((0.02 * rng.normal(size=D)).astype(np.float32)).cuda()
    small = big[:6240].contiguous()
    y_big = sra.layer_norm(big, g, b)
    y_small = sra.layer_norm(small, g, b)
    assert torch.equal(y_big[:6240], y_small)


# ------------------------------------------------------------------ attention
@pytest.mark.parametrize("lens,H", [([13], 4), ([104, 104, 104, 78], 20), ([1, 5, 64, 65, 100, 128], 3),
                                    ([1, 5, 64, 65, 100, 128, 129], 3), ([17, 32, 33], 2), ([1500, 1500], 12)])
def test_attention(lens, H):
    rng = np.random.default_rng(sum(lens) + H)
    T = sum(lens)
    qkv = _bf16(rng.normal(size=(T, 3 * H * 64)))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    got = sra.attention(qkv.cuda(), torch.from_numpy(cu).cuda(), H).float().cpu().numpy()
    q = qkv.float().numpy()
    d = H * 64
    ref = oracle.attention_windows(q[:, :d], q[:, d:2 * d], q[:, 2 * d:], cu, H)
    err = np.abs(got - ref).max()
    assert err <= 2e-2, err
    # rows of a one-token window copy the value row
    if lens[0] == 1:
        np.testing.assert_allclose(got[0], q[0, 2 * d:], atol=1e-2)


@pytest.mark.parametrize("case", ["windows_16x30s", "ragged"])
def test_attention_many_items_per_block(case):
    """Many more (segment, head) blocks than fit on the GPU at once: the
    16 x 30 s window layout (64 windows x 20 heads, several waves of blocks)
    and a ragged mix of 150 segments of 1..128 tokens, element by element
    against the oracle, and the same bits from a second call."""
    rng = np.random.default_rng(11 if case == "ragged" else 12)
    if case == "ragged":
        lens, H = [int(v) for v in rng.integers(1, 129, size=150)], 7
    else:
        lens, H = [104, 104, 104, 78] * 16, 20
    T = sum(lens)
    qkv = _bf16(rng.normal(size=(T, 3 * H * 64)))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    got = sra.attention(qkv.cuda(), torch.from_numpy(cu).cuda(), H).float().cpu().numpy()
    q = qkv.float().numpy()
    d = H * 64
    ref = oracle.attention_windows(q[:, :d], q[:, d:2 * d], q[:, 2 * d:], cu, H)
    assert np.abs(got - ref).max() <= 2e-2
    # a second call on the same inputs gives the same bits
    again = sra.attention(qkv.cuda(), torch.from_numpy(cu).cuda(), H).float().cpu().numpy()
    assert np.array_equal(got, again)


def test_attention_large_orthogonal_rows():
    """Head 0 has query and key rows of norm 300 along different axes, so
    their scores come only from small components and sit far below the
    product of the norms (a softmax shifted by a norm bound instead of the
    row maximum would underflow here).  Head 1 is ordinary; both are
    compared with the oracle element by element."""
    rng = np.random.default_rng(21)
    H, lens = 2, [104, 104, 57, 1]
    T, d = sum(lens), 2 * 64
    q = rng.normal(size=(T, d)) * 0.6
    k = rng.normal(size=(T, d)) * 0.6
    q[:, :64] *= 0.05
    k[:, :64] *= 0.05
    q[:, 0] = 300.0
    k[:, 1] = 300.0
    v = rng.normal(size=(T, d))
    qkv = _bf16(np.concatenate([q, k, v], axis=1))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    got = sra.attention(qkv.cuda(), torch.from_numpy(cu).cuda(), H).float().cpu().numpy()
    x = qkv.float().numpy()
    ref = oracle.attention_windows(x[:, :d], x[:, d:2 * d], x[:, 2 * d:], cu, H)
    assert np.isfinite(got).all()
    assert np.abs(got - ref).max() <= 2e-2


@pytest.mark.parametrize("lens,H", [([200, 300, 257, 1], 2), ([1500], 3), ([130, 129, 384, 385], 1)])
def test_attention_long_segments(lens, H):
    """Segments longer than one 128-key tile run on the flash kernel (online
    softmax over key tiles, O in tensor memory)."""
    rng = np.random.default_rng(sum(lens) * 7 + H)
    T = sum(lens)
    qkv = _bf16(rng.normal(size=(T, 3 * H * 64)))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    got = sra.attention(qkv.cuda(), torch.from_numpy(cu).cuda(), H).float().cpu().numpy()
    q = qkv.float().numpy()
    d = H * 64
    ref = oracle.attention_windows(q[:, :d], q[:, d:2 * d], q[:, 2 * d:], cu, H)
    assert np.abs(got - ref).max() <= 2e-2


def test_attention_long_segment_rescale():
    """Keys whose scores grow tile after tile: the running maximum moves by
    more than the lazy-rescale threshold several times within a row."""
    rng = np.random.default_rng(3)
    H, L = 2, 1000
    q = rng.normal(size=(L, H * 64)) * 0.6
    k = rng.normal(size=(L, H * 64)) * 0.6
    k *= (1.0 + np.arange(L) // 128)[:, None] * 1.5      # scores scale up with the key tile
    v = rng.normal(size=(L, H * 64))
    qkv = _bf16(np.concatenate([q, k, v], axis=1))
    cu = np.array([0, L], dtype=np.int32)
    got = sra.attention(qkv.cuda(), torch.from_numpy(cu).cuda(), H).float().cpu().numpy()
    x = qkv.float().numpy()
    d = H * 64
    ref = oracle.attention_windows(x[:, :d], x[:, d:2 * d], x[:, 2 * d:], cu, H)
    assert np.abs(got - ref).max() <= 2e-2


# ------------------------------------------------------------------ GELU
def test_gelu_within_published_bound():
    # The device GELU is the tanh form 0.5 x (1 + tanh(sqrt(2/pi)(x + 0.044715 x^3)))
    # (Hendrycks & Gimpel): within 4.8e-4 of the exact x Phi(x) (the form's own
    # maximum is 4.74e-4, checked on the CPU below), plus 0.5 |x| times the
    # hardware tanh's relative error (<= 2^-10.98), plus fp32 rounding.  An odd
    # length sends the last element through the scalar form, the rest through
    # the packed pair form.
    x = np.concatenate([np.linspace(-12, 12, 2_000_001), [0.0, -0.0, 1e-30, -1e-30, 40.0, -40.0]]).astype(np.float32)
    assert len(x) % 2 == 1
    xd = x.astype(np.float64)
    form = 0.5 * xd * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (xd + 0.044715 * xd ** 3)))
    ref = oracle.gelu(xd)
    assert np.abs(form - ref).max() <= 4.8e-4
    got = sra.gelu(torch.from_numpy(x).cuda()).cpu().numpy().astype(np.float64)
    err = np.abs(got - ref)
    bound = 4.8e-4 + (0.5 * 2.0 ** -10.98 + 2.0 ** -22) * np.abs(x) + 2.0 ** -22 * np.abs(ref)
    assert (err <= bound).all(), (err.max(), (err / np.maximum(bound, 1e-300)).max())
    assert got[-2] == 40.0 and abs(got[-1]) == 0.0
    assert np.all(np.isfinite(got))


# ------------------------------------------------------------------ bounded waits
def test_wait_probe_times_out_and_context_survives():
    st = sra.wait_probe(50_000_000)  # 50 ms
    assert st == 6
    # the context is still usable afterwards
    x = torch.ones(1000, device="cuda")
    assert float(x.sum().item()) == 1000.0
    m = sra.log_mel(torch.from_numpy(synth.pcm_clip(16000, 1)[None]).cuda(), 128)
    assert torch.isfinite(m).all()
