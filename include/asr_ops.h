/*
 * asr_ops.h -- kernel-level entry points of the ASR encoder library.
 *
 * Each call runs one stage of the forward pass with exactly the kernel that
 * asr_enc_forward launches for it, on caller-owned device buffers, so that
 * every stage can be checked on its own.  Conventions as in asr_enc.h
 * (device pointers, stream as void*, asr_status return, asynchronous).
 */
#ifndef ASR_OPS_H
#define ASR_OPS_H

#include "asr_enc.h"

#ifdef __cplusplus
extern "C" {
#endif
#if defined(__GNUC__)
#pragma GCC visibility push(default)
#endif

/* Log-mel front-end of a batch of clips ("MOSS-Transcribe-preview-2B-GGUF",
 * Architecture "Audio" row; Non-obvious gotchas on the trailing frame):
 * periodic Hann(400), centred reflect-padded frames every 160 samples,
 * |DFT|^2 of 201 bins, trailing frame dropped, Slaney mel filterbank (0-8 kHz),
 * log10(max(., 1e-10)), clamp at (clip max - 8), then (x + 4) / 4.
 *  pcm   device float32 [batch, n_samples]; n_samples % 160 == 0, > 200.
 *  mel   device float32 [batch, n_mels, n_samples/160] (normalised).
 *  ws    device scratch of >= asr_op_log_mel_ws_size(batch) bytes, 256-byte
 *        aligned: the per-clip maxima and the FFT / filterbank tables, which
 *        every call rebuilds on the device (one small kernel, no host copy).
 * n_mels: 1..128. */
size_t asr_op_log_mel_ws_size(int batch);
asr_status asr_op_log_mel(const float* pcm, int64_t n_samples, int batch, int n_mels, float* mel,
                          void* ws, size_t ws_bytes, void* stream);

/* Log-mel front-end that allocates no memory.  The pages have no
 * counterpart: this entry point exists for callers that must not call
 * cudaMalloc -- for example a plugin inside a host application that owns all
 * device memory, or a real-time audio thread, where an allocation would
 * stall on an implicit device synchronisation.  It computes exactly what
 * asr_op_log_mel computes (same kernels, same tables, bit-identical output),
 * but its scratch (the per-clip maxima and the FFT / filterbank tables,
 * about 31 KB) is a fixed array inside the library: every GPU that loads the
 * library holds it until the process exits.
 *  pcm, n_samples, n_mels, mel: as for asr_op_log_mel.
 *  batch: 1 .. 4096 clips; larger batches return ASR_E_UNSUPPORTED.
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  Each call then enqueues on `stream` a kernel
 * that rebuilds the tables for its n_mels, a memset that clears the maxima,
 * and the log-mel kernels; nothing is copied from the host and the calling
 * thread does not wait for the device.  All calls share the one array and it
 * keeps the last call's contents, so calls whose GPU work overlaps
 * (different streams, not ordered) race and must not be issued; calls on
 * one stream are ordered and may use different n_mels. */
asr_status asr_op_log_mel_noalloc(const float* pcm, int64_t n_samples, int batch, int n_mels, float* mel,
                                  void* stream);

/* Dense layer on the tcgen05 GEMM engine: acc = X W^T (fp32 accumulate in
 * tensor memory), then the epilogue.
 *  x     device bf16 [M, K] row-major;  w  device bf16 [N, K] row-major.
 *  bias  device float32 [N] or NULL.
 *  epi   ASR_EPI_BF16       y bf16 [M, N] = acc + bias
 *        ASR_EPI_BF16_GELU  y bf16 [M, N] = GELU(acc + bias), the GELU of asr_op_gelu
 *                           (tanh form, |error| <= 4.8e-4 + 2.5e-4 |x|)
 *        ASR_EPI_F32_RESID  y f32  [M, N] += acc + bias           (in place)
 *        ASR_EPI_F32        y f32  [M, N] = acc + bias
 *        ASR_EPI_SWIGLU     y bf16 [M, N/2]: W rows interleaved in blocks of
 *                           16 (gate rows 16j..16j+15, then the matching up
 *                           rows), y[:, 16j+i] = SiLU(gate) * up
 * Limits: K % 8 == 0, N % 16 == 0, M >= 1.  ws: device scratch, caller-owned,
 * at least 256 bytes (device status word).  With asr_op_linear_ws_size()
 * bytes (status word and one flag per SM and epilogue warp of the current
 * device) the residual epilogue on CTA-pair tiles runs stream-K: the
 * (tile, k-block) work is split evenly over the SM pairs, and of a tile cut
 * in two the trailing part's sum reaches y before the leading part's, so
 * results are deterministic.  Smaller scratch runs whole tiles.
 * tile_n: output tile of one SM, 128 x tile_n (256, 160, 128 or 64; 160 needs
 * N % 160 == 0), or of a CTA pair (two SMs, tcgen05 cta_group::2),
 * 256 x -tile_n (-256 or -128); 0 = chosen from M, N and the SM count as in
 * the forward pass. */
enum { ASR_EPI_BF16 = 0, ASR_EPI_BF16_GELU = 1, ASR_EPI_F32_RESID = 2, ASR_EPI_F32 = 3,
       ASR_EPI_SWIGLU = 4 };
size_t asr_op_linear_ws_size(void);
asr_status asr_op_linear(const void* x, const void* w, const float* bias, int64_t M, int N, int K,
                         int epi, int tile_n, void* y, void* ws, size_t ws_bytes, void* stream);

/* Residual dense layer and the LayerNorm of the updated rows in one launch
 * of the CTA-pair engine (the epilogue of the encoder's out-projection and
 * fc2; "Audio encoder": pre-norm blocks):
 *   y[M, N] += X W^T + bias                                  (f32, in place)
 *   h[M, N]  = (y - mean) / sqrt(var + eps) * gamma + beta   (bf16; mean and
 *              biased variance over each updated row of y)
 * The update of y is computed exactly as by ASR_EPI_F32_RESID (same adds in
 * the same order); the statistics combine per-tile partial means and sums of
 * squared deviations (Chan, Golub and LeVeque's pairwise update).
 *  x bf16 [M, K] row-major;  w bf16 [N, K];  bias, gamma, beta f32 [N].
 *  Limits: M >= 1, K % 128 == 0, N % 32 == 0, ceil(N / 256) <= the CTA pairs
 *  the device can hold at once (74 on a B200), 16-byte aligned pointers.
 *  ws: device scratch of at least asr_op_linear_resid_ln_ws_size(M, N)
 *  bytes (status word, one counter per 32 rows, and per row two 16-byte
 *  partial statistics per 256 columns); the call clears what it needs with
 *  a memset on `stream`.  ASR_E_UNSUPPORTED when the shape is outside the
 *  limits; a statistics wait that runs out (bounded, seconds) is reported by
 *  the status word like the engine's other waits. */
size_t asr_op_linear_resid_ln_ws_size(int64_t M, int N);
asr_status asr_op_linear_resid_ln(const void* x, const void* w, const float* bias, const float* gamma,
                                  const float* beta, float eps, int64_t M, int N, int K, float* y, void* h,
                                  void* ws, size_t ws_bytes, void* stream);

/* The same engine with fp32 operands multiplied as tf32 (tcgen05 kind::tf32:
 * the tensor cores read each fp32 operand's sign, exponent and top 10
 * mantissa bits) and fp32 accumulation; the path of geometries with fp32
 * weights.
 *  x  device float32 [M, K];  w  device float32 [N, K];  y device float32.
 *  epi: ASR_EPI_F32 (y = acc + bias), ASR_EPI_BF16_GELU (y = GELU(acc +
 *  bias), fp32 output), ASR_EPI_F32_RESID (y += acc + bias) or ASR_EPI_SWIGLU
 *  (y [M, N/2] fp32, rows interleaved as for asr_op_linear).
 *  tile_n: 0, 256, 128 or 64 (one-SM tiles).  Limits: K % 4 == 0 (16-byte
 *  rows), N % 16 == 0.  ws: >= 256 bytes (device status word). */
asr_status asr_op_linear_tf32(const float* x, const float* w, const float* bias, int64_t M, int N, int K, int epi,
                              int tile_n, float* y, void* ws, size_t ws_bytes, void* stream);

/* LayerNorm over the last axis: y = (x - mean) / sqrt(var + eps) * g + b,
 * x device float32 [M, D], g/b device float32 [D], y device bf16 [M, D]
 * (out_f32 == 0) or float32 (out_f32 != 0).  D must be a multiple of 128 and
 * at most 2048 (ASR_E_INVAL otherwise); M >= 1. */
asr_status asr_op_layer_norm(const float* x, const float* g, const float* b, int64_t M, int D,
                             float eps, void* y, int out_f32, void* stream);

/* Windowed / full attention over segments: for each segment [cu[j], cu[j+1])
 * and head h, softmax(Q K^T / 8) V, with Q, K, V read from
 * qkv device bf16 [T, 3*H*64] (columns: q heads, k heads, v heads) and the
 * result written to out device bf16 [T, H*64].  cu: device int32 [n_seg+1].
 * max_seg: the longest segment.  head_dim 64.  Segments of at most 128
 * tokens run on the tcgen05 kernel (one block per segment and head), longer
 * ones on a flash-style kernel.  ws: device scratch of
 * >= asr_op_attention_ws_size() bytes (device status word). */
size_t asr_op_attention_ws_size(void);
asr_status asr_op_attention(const void* qkv, const int32_t* cu, int n_seg, int max_seg, int64_t T,
                            int H, void* out, void* ws, size_t ws_bytes, void* stream);

/* The GELU every kernel applies (bias-free): y[i] = GELU(x[i]) in the tanh
 * form 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))) (Hendrycks & Gimpel),
 * with tanh from the hardware tanh.approx.f32: |y - x Phi(x)| <= 4.8e-4 (the
 * form) + 2.5e-4 |x| (the approximate tanh), below the rounding of a bf16
 * output for |x| >= 0.5.  x, y: device float32 [n]. */
asr_status asr_op_gelu(const float* x, float* y, int64_t n, void* stream);

/* Bounded-wait self-check: launches one kernel that waits on a shared-memory
 * barrier that nothing ever completes, gives up after limit_ns nanoseconds
 * of device time, writes 1 to *status_dev (device int32) and returns
 * normally.  It shows that a stalled device wait ends with a status the host
 * can read while the CUDA context stays usable. */
asr_status asr_op_wait_probe(int64_t limit_ns, int* status_dev, void* stream);

#if defined(__GNUC__)
#pragma GCC visibility pop
#endif
#ifdef __cplusplus
}
#endif
#endif /* ASR_OPS_H */
