/*
 * asr_enc.h -- C ABI of the B200 (sm_100a) ASR audio-encoder forward pass.
 *
 * The operation: 16 kHz mono PCM -> log-mel -> conv stem -> pre-LN
 * transformer tower with windowed (block-diagonal) or full attention ->
 * encoder head -> SwiGLU adapter, as described by
 *   "MOSS-Transcribe-preview-2B-GGUF", Architecture table (rows "Audio
 *   encoder", "Conv front-end", "Encoder head", "Adapter", "Audio") and
 *   Non-obvious gotchas (trailing STFT frame dropped: n_samples/hop frames);
 * and, for the full-attention variant with a Conv1D stem, by
 *   "CrisperWhisper -> ONNX (with cross-attentions)", What this exports
 *   instead (whisper-small geometry) and Results (1500 encoder frames per
 *   30 s window).
 *
 * Conventions for every entry point:
 *   - Plain C types only.  Device pointers are CUDA device addresses on the
 *     current device; `stream` is a cudaStream_t passed as void* (NULL = the
 *     legacy default stream).
 *   - Nothing is thrown across the ABI; each call returns an asr_status.
 *     On failure, asr_enc_last_error() returns a message (per handle, or the
 *     process-wide one when the handle is NULL).
 *   - Calls are asynchronous with respect to the host unless stated; the
 *     library synchronises only where a call says it reads device memory
 *     back (asr_enc_sync_status, asr_enc_forward_host).
 *   - The caller owns every buffer it passes.  The handle owns the repacked
 *     weights it obtained through the caller's allocator at create time.
 */
#ifndef ASR_ENC_H
#define ASR_ENC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif
#if defined(__GNUC__)
#pragma GCC visibility push(default)
#endif

typedef struct asr_enc asr_enc; /* opaque, library-owned */

typedef enum {
  ASR_OK = 0,
  ASR_E_INVAL = 1,          /* bad argument: NULL pointer, bad geometry or size */
  ASR_E_UNSUPPORTED = 2,    /* well-formed but outside what this build implements */
  ASR_E_NOMEM = 3,          /* the allocator callback returned NULL */
  ASR_E_CUDA = 4,           /* a CUDA runtime/driver call failed (message has the name) */
  ASR_E_WORKSPACE = 5,      /* workspace NULL or smaller than asr_enc_workspace_size() */
  ASR_E_DEVICE_TIMEOUT = 6  /* a bounded device-side wait gave up (see asr_enc_sync_status) */
} asr_status;

enum { ASR_STEM_CONV2D_CHUNKED = 0, ASR_STEM_CONV1D = 1 };
enum { ASR_POS_PER_CHUNK = 0, ASR_POS_GLOBAL = 1 };
enum { ASR_DTYPE_BF16 = 0, ASR_DTYPE_F32 = 1, ASR_DTYPE_F16 = 2 };

/* Encoder geometry.  Field meanings:
 *  stem           ASR_STEM_CONV2D_CHUNKED: 3 x Conv2D k3 s2 p1 (1->C->C->C) + GELU
 *                 applied per chunk of chunk_frames mel frames, then conv_out
 *                 (C*n_mels/8 -> d_model, no bias) ("Conv front-end" row).
 *                 ASR_STEM_CONV1D: Conv1D k3 s1 p1 (n_mels->d) + GELU, Conv1D
 *                 k3 s2 p1 (d->d) + GELU (whisper-small geometry).
 *  n_mels, n_fft, hop   128|80, 400, 160 ("Audio" row).  Only n_fft 400 / hop 160.
 *  chunk_frames   100 (conv2d stem only; 0 otherwise).
 *  conv_ch        Conv2D channels C (480); ignored by the Conv1D stem.
 *  d_model, n_heads, head_dim, d_ffn, n_layers   tower shape; head_dim must be 64.
 *  window_tokens  attention window in tokens (104); 0 = full attention per clip.
 *  pos_mode       ASR_POS_PER_CHUNK (positions restart each chunk) or ASR_POS_GLOBAL.
 *  proj1_out, proj2_out        encoder head widths; 0 = absent (final LN only).
 *  adapter_hidden, adapter_out SwiGLU adapter widths; 0 = absent.
 *  ln_eps         LayerNorm epsilon.
 *  dtype          the weights' type, which sets the arithmetic of every GEMM:
 *                 ASR_DTYPE_BF16  bf16 weights, bf16 activations between the
 *                                 GEMMs, tcgen05 kind::f16, fp32 accumulation;
 *                 ASR_DTYPE_F16   f16 weights and activations (the F16 variant
 *                                 of the pages' GGUF builds), kind::f16;
 *                 ASR_DTYPE_F32   fp32 weights and activations, kind::tf32
 *                                 GEMMs, attention in fp32 on the CUDA cores.
 *                 The residual stream, softmax, LayerNorm statistics and the
 *                 log-mel are fp32 in every case.
 */
typedef struct {
  int stem;
  int n_mels, n_fft, hop, chunk_frames;
  int conv_ch, d_model, n_heads, head_dim, d_ffn, n_layers;
  int window_tokens;
  int pos_mode;
  int proj1_out, proj2_out, adapter_hidden, adapter_out;
  float ln_eps;
  int dtype;
} asr_geometry;

/* Device allocator supplied by the caller (e.g. a PyTorch caching allocator).
 * alloc returns a device pointer aligned to >= 256 bytes or NULL. */
typedef void* (*asr_alloc_fn)(void* ctx, size_t bytes);
typedef void (*asr_free_fn)(void* ctx, void* ptr);

/* ---- weights ------------------------------------------------------------
 * Weights are passed as an array of device pointers in a fixed name order.
 * asr_enc_weight_count() gives the count; asr_enc_weight_info() the name,
 * rank and shape of entry i.  Matrices are [out, in] row-major (torch Linear
 * layout); Conv2D kernels [out, in, kh(freq), kw(time)]; Conv1D kernels
 * [out, in, k]; biases and LayerNorm gain/shift are vectors.  Every tensor
 * is of the geometry's dtype.  Order: conv1.w conv1.b conv2.w conv2.b
 * [conv3.w conv3.b conv_out.w] then per layer l: ln1.g ln1.b q.w q.b k.w k.b
 * v.w v.b o.w o.b ln2.g ln2.b fc1.w fc1.b fc2.w fc2.b, then ln_post.g
 * ln_post.b [proj1.w proj1.b proj2.w proj2.b] [adapter.gate.w adapter.up.w
 * adapter.down.w].  Returns -1 for an invalid geometry. */
int asr_enc_weight_count(const asr_geometry* g);
/* name: static string owned by the library; shape: up to 4 extents. */
asr_status asr_enc_weight_info(const asr_geometry* g, int i, const char** name, int* ndim,
                               int64_t shape[4]);

/* ---- geometry queries (host only, bit-exact) ----------------------------- */

/* Tokens per clip of n_samples (> n_fft / 2): frames F = floor(n_samples /
 * hop) (trailing STFT frame dropped); conv2d stem: the frames are cut into
 * chunks of chunk_frames, the last one short when F is not a multiple, and a
 * chunk of L frames gives ceil(ceil(ceil(L / 2) / 2) / 2) tokens (13 for 100);
 * conv1d stem: frames after k3 s1 p1 then k3 s2 p1 (ceil(F / 2)).  Returns -1
 * for n_samples <= n_fft / 2 or an invalid geometry. */
int64_t asr_enc_tokens(const asr_geometry* g, int64_t n_samples);

/* Attention-window partition of a batch of `batch` clips of n_samples each,
 * as cumulative token offsets cu[0..n] (int32, cu[0]=0, cu[n]=batch*tokens).
 * Windows tile each clip from its first token in steps of window_tokens, the
 * last one short; window_tokens==0 gives one window per clip.  *n is in/out:
 * capacity of cu in entries on input (n+1 needed), window count on output.
 * With cu==NULL only the count is returned. */
asr_status asr_enc_windows(const asr_geometry* g, int64_t n_samples, int batch, int32_t* cu,
                           int* n);

/* ---- handle lifecycle ---------------------------------------------------- */

/* Validate the geometry, then copy and repack the weights (fused QKV rows,
 * permuted conv_out columns, conv kernels in tap-major/channel-minor order,
 * fp32 bias and LayerNorm vectors) into device buffers obtained from
 * `alloc` (cudaMalloc when alloc is NULL), and build the weight TMA
 * descriptors.  `weights` points to asr_enc_weight_count(g) device pointers.
 * Work is enqueued on `stream` and completed before return.
 * Limits: n_mels 1..128, n_fft 400, hop 160, head_dim 64 with n_heads * 64 ==
 * d_model, d_model a multiple of 128 and <= 2048, d_ffn a multiple of 64,
 * conv_ch a multiple of 8 and <= 512, proj1_out % 64 == 0, proj2_out % 128 == 0
 * and <= 2048, adapter widths multiples of 16; otherwise ASR_E_UNSUPPORTED.
 * Every CUDA runtime call made here is checked: a failed copy or launch
 * returns ASR_E_CUDA naming the call, and nothing is left allocated. */
asr_status asr_enc_create(const asr_geometry* g, const void* const* weights, int n_weights,
                          asr_alloc_fn alloc, asr_free_fn free_fn, void* alloc_ctx, void* stream,
                          asr_enc** out);

/* Release everything the handle owns (through free_fn).  NULL is a no-op.
 * The caller must ensure no forward using the handle is still running. */
void asr_enc_destroy(asr_enc* e);

/* Bytes of workspace a forward of `batch` clips of n_samples needs
 * (0 on invalid sizes). */
size_t asr_enc_workspace_size(const asr_enc* e, int64_t n_samples, int batch);

/* ---- forward ------------------------------------------------------------- */

/* Run the whole forward on `stream`.
 *  pcm         device float32 [batch, n_samples], row-major.
 *  n_samples   per clip, > n_fft / 2.  Conv1d stem: an even number of hops
 *              (ASR_E_UNSUPPORTED otherwise).  Conv2d stem: any length; a
 *              clip whose frames are not whole chunks gets a short last
 *              chunk (see asr_enc_forward_varlen).
 *  out         device float32 [batch, T, D_out], T = asr_enc_tokens(),
 *              D_out = adapter_out, else proj2_out, else d_model.
 *  out_tokens  optional host pointer; receives T.
 *  workspace   device buffer of >= asr_enc_workspace_size() bytes,
 *              256-byte aligned; the forward may overwrite all of it.
 * Asynchronous.  Bounded device waits that give up set the handle's device
 * status word; read it with asr_enc_sync_status(). */
asr_status asr_enc_forward(asr_enc* e, const float* pcm, int64_t n_samples, int batch, float* out,
                           int64_t* out_tokens, void* workspace, size_t ws_bytes, void* stream);

/* Variable-length batch (conv2d stem only; ASR_E_UNSUPPORTED otherwise):
 * clip b has n_samples[b] samples (host int64 array, each > n_fft / 2).
 *  pcm         device float32, the clips packed back to back (sum of
 *              n_samples floats).
 *  out         device float32 [sum of T_b, D_out]: each clip's token rows,
 *              packed in clip order, T_b = asr_enc_tokens(g, n_samples[b]).
 *  out_tokens  optional host int64 [batch]; receives T_b.
 *  workspace   >= asr_enc_workspace_size_varlen() bytes, 256-byte aligned.
 * Each clip has its own log-mel maximum and attention windows; a clip's
 * last chunk holds its remaining frames (computed as a zero-padded whole
 * chunk whose conv outputs past the short chunk's own lengths are zeroed, so
 * each result equals the short chunk's convolution) and gives fewer tokens,
 * whose positions restart at 0 like every chunk's.  The mel tap is not
 * available for these batches. */
size_t asr_enc_workspace_size_varlen(const asr_enc* e, const int64_t* n_samples, int batch);
asr_status asr_enc_forward_varlen(asr_enc* e, const float* pcm, const int64_t* n_samples, int batch, float* out,
                                  int64_t* out_tokens, void* workspace, size_t ws_bytes, void* stream);

/* Same as asr_enc_forward but with HOST buffers: copies pcm (host float32
 * [batch, n_samples]; page-locked for full speed) into the workspace, runs
 * the forward and copies the result back into host `out` ([batch, T,
 * D_out]).  Synchronises `stream` and returns the device status. */
asr_status asr_enc_forward_host(asr_enc* e, const float* pcm_host, int64_t n_samples, int batch,
                                float* out_host, int64_t* out_tokens, void* workspace,
                                size_t ws_bytes, void* stream);
/* Host-buffer form of asr_enc_forward_varlen (packed host pcm and out). */
asr_status asr_enc_forward_host_varlen(asr_enc* e, const float* pcm_host, const int64_t* n_samples, int batch,
                                       float* out_host, int64_t* out_tokens, void* workspace, size_t ws_bytes,
                                       void* stream);

/* Synchronise the stream of the last forward and read the device status
 * word: ASR_OK, or ASR_E_DEVICE_TIMEOUT if a bounded wait gave up. */
asr_status asr_enc_sync_status(asr_enc* e);

/* ---- per-stage taps (debug / parity) --------------------------------------
 * With taps enabled (mask of 1<<stage), the forward also copies the listed
 * stage tensors into the workspace (asr_enc_workspace_size grows
 * accordingly), and asr_enc_tap copies the last forward's tensor to `dst`
 * (device, float32) after checking dst_bytes.  Stages and shapes:
 *  ASR_TAP_MEL      [batch, n_mels, n_samples/hop]  normalised log-mel
 *  ASR_TAP_STEM     [batch*T, d_model]  after the stem and positions
 *  ASR_TAP_LAYER0   [batch*T, d_model]  residual stream after layer 0
 *  ASR_TAP_ENCODER  [batch*T, d_model]  after the last layer (before ln_post)
 *  ASR_TAP_HEAD     [batch*T, proj2_out] head output (adapter input)
 * The workspace must not be reused between the forward and the tap call. */
enum { ASR_TAP_MEL = 0, ASR_TAP_STEM = 1, ASR_TAP_LAYER0 = 2, ASR_TAP_ENCODER = 3, ASR_TAP_HEAD = 4,
       ASR_TAP_COUNT = 5 };
asr_status asr_enc_set_taps(asr_enc* e, unsigned mask);
asr_status asr_enc_tap(asr_enc* e, int stage, float* dst, size_t dst_bytes, void* stream);

/* ---- CUDA-graph replay -------------------------------------------------------
 * A uniform forward (asr_enc_forward / asr_enc_forward_host) is recorded as a
 * CUDA graph on the encoder's own stream the first time a given set of
 * (pcm, out, workspace) pointers, n_samples, batch and tap mask is seen, and
 * the graph is launched on the caller's stream then and on every later call
 * with the same set (one launch instead of one per kernel; results are
 * bit-identical to the direct launches).  A new set records a new graph and
 * drops the old one.  Variable-length batches, profiling, and a caller whose
 * stream is itself being captured launch the kernels directly.  If recording
 * fails the encoder falls back to direct launches for good.  The data behind
 * the pointers may change between calls; the pointers may not be freed while
 * the encoder may still replay a graph that uses them (a later call with other
 * pointers, asr_enc_set_graphs(e, 0) or asr_enc_destroy releases it).
 * asr_enc_set_graphs(e, 0) turns recording off (and drops the graph); 1 turns
 * it back on.  Default: on. */
asr_status asr_enc_set_graphs(asr_enc* e, int enable);

/* ---- LayerNorm epilogue ------------------------------------------------------
 * With 16-bit weights whose shapes allow it (d_model and d_ffn multiples of
 * 128, d_model a multiple of 32), the fc2 GEMM of every block also computes
 * the LayerNorm that reads its residual update ("Audio encoder": pre-norm
 * blocks, each sub-layer's input is the LayerNorm of the residual stream):
 * the next block's first LayerNorm, or the head's LayerNorm after the last
 * block when there is a projection head.  The GEMM's epilogue adds its tile
 * to the fp32 residual stream, publishes the rows' partial mean / sum of
 * squared deviations, waits (bounded) for the other tiles of the same rows,
 * and writes the normalised 16-bit rows; the separate LayerNorm launch goes
 * away.  (The attention out-projection keeps its separate LayerNorm: with
 * K = d_model its mainloop is shorter than that epilogue.)  The residual
 * stream is computed with the same additions as the unfused path; the
 * LayerNorm outputs differ by the summation order of the statistics (well
 * inside the encoder's tolerance), and so does everything downstream.
 * asr_enc_set_ln_fusion(e, 1) turns it on, 0 off (the separate LayerNorm
 * kernels run; either call drops a recorded graph).  Default: off — on one
 * B200 the separate single-wave LayerNorm launches make the 16 x 30 s
 * forward about 0.17 ms faster than the fused epilogue.
 * asr_enc_ln_fusion reports whether forwards use it (*active = 1) or not. */
asr_status asr_enc_set_ln_fusion(asr_enc* e, int enable);
asr_status asr_enc_ln_fusion(const asr_enc* e, int* active);

/* ---- kernel timing (profiling) --------------------------------------------
 * asr_enc_profile(e, 1) makes every later forward bracket each of its kernel
 * launches with CUDA events on the forward's stream (small extra cost; do not
 * enable inside CUDA-graph capture).  asr_enc_profile_read synchronises the
 * last forward's stream and returns per-stage totals: up to max entries of
 * (static name, milliseconds, launches); the return value is the number of
 * stages written, or -1 on error.  asr_enc_last_launches returns how many
 * kernels the last forward launched (always counted). */
asr_status asr_enc_profile(asr_enc* e, int enable);
int asr_enc_profile_read(asr_enc* e, int max, const char** names, double* ms, int* launches);
int asr_enc_last_launches(const asr_enc* e);

/* ---- audio injection --------------------------------------------------------
 * The LLM input embeddings of a tokenised prompt with the audio spliced in
 * ("MOSS-Transcribe-preview-2B-GGUF", Architecture table, "Audio injection":
 * the placeholder positions' token embeddings are replaced by the adapter
 * output frames; "Prompt": the audio sits between <|audio_start|> and
 * <|audio_end|> of a ChatML user turn).
 *  ids          device int32 [n_ids], n_ids >= 1: the prompt's token ids (a
 *               batch of prompts is passed as one packed sequence).
 *  placeholder  the id of the audio placeholder token.
 *  table        device [vocab, dim] token-embedding table of table_dtype
 *               (ASR_DTYPE_BF16, ASR_DTYPE_F16 or ASR_DTYPE_F32).
 *  frames       device float32 [n_frames, dim]: adapter output rows (the
 *               forward's output of each clip, clips in prompt order).
 *  out          device [n_ids, dim] of out_dtype: row i is frames[r] when
 *               ids[i] == placeholder, r being the number of placeholders
 *               before i, else table[ids[i]]; values are converted to
 *               out_dtype with round-to-nearest-even (same-type rows are
 *               copied bit for bit).
 *  ws           device scratch of >= asr_splice_ws_size(n_ids) bytes,
 *               256-byte aligned; its first int32 is the status word:
 *               0 ok, 1 an id outside [0, vocab) (that row is zero), 2 the
 *               placeholder count differs from n_frames (rows without a
 *               frame are zero).  Asynchronous; asr_splice_check()
 *               synchronises the stream and turns the word into ASR_OK or
 *               ASR_E_INVAL. */
size_t asr_splice_ws_size(int64_t n_ids);
asr_status asr_splice_embeddings(const int32_t* ids, int64_t n_ids, int32_t placeholder, const void* table,
                                 int vocab, int table_dtype, const float* frames, int64_t n_frames, int dim,
                                 void* out, int out_dtype, void* ws, size_t ws_bytes, void* stream);
asr_status asr_splice_check(const void* ws, void* stream);

/* ---- streaming ---------------------------------------------------------------
 * Live input, encoded one attention window at a time (the windows are
 * independent: "MOSS-Transcribe-preview-2B-GGUF", Architecture, "Audio
 * encoder", windowed block-diagonal attention).  Conv2d stem with
 * window_tokens a whole number of chunks' tokens only (ASR_E_UNSUPPORTED
 * otherwise).  Window j covers the stream's mel frames [j WF, (j + 1) WF),
 * WF = window_tokens / (tokens per chunk) * chunk_frames (800 frames = 8 s for
 * the 104-token windows of 100-frame chunks).  Its frames are the centred
 * STFT frames of the whole stream (reflection only at the stream's start and
 * end), and its log-mel is normalised by the maximum over its own frames --
 * the offline forward normalises by the clip's maximum instead, which a live
 * stream cannot know in advance.  A window is encoded as soon as the samples
 * its last frame reads have arrived ((j + 1) WF - 1) hop + n_fft / 2 samples).
 *  asr_stream_create: state on the encoder `e` (which must outlive it); its
 *      sample buffer comes from the encoder's allocator and grows as needed.
 *  asr_stream_push: appends n device float32 samples (n >= 0), encodes every
 *      window that became ready and writes their rows, packed in window order,
 *      to device float32 out [*out_rows, D_out] (out_cap_rows rows
 *      available; asr_stream_window_tokens() rows per window); the workspace
 *      must hold asr_stream_workspace_size(e, windows) for the number of
 *      windows that become ready.  Asynchronous on `stream`; use one stream
 *      per stream object.
 *  asr_stream_finish: encodes the remaining frames as a last, possibly
 *      short window (a short last chunk as in asr_enc_forward_varlen); after
 *      it the stream takes no more samples.  Needs > n_fft / 2 samples in all. */
typedef struct asr_stream asr_stream;
int64_t asr_stream_window_tokens(const asr_enc* e);
size_t asr_stream_workspace_size(const asr_enc* e, int windows);
asr_status asr_stream_create(asr_enc* e, asr_stream** out);
asr_status asr_stream_push(asr_stream* s, const float* pcm, int64_t n, float* out, int64_t out_cap_rows,
                           int64_t* out_rows, void* ws, size_t ws_bytes, void* stream);
asr_status asr_stream_finish(asr_stream* s, float* out, int64_t out_cap_rows, int64_t* out_rows, void* ws,
                             size_t ws_bytes, void* stream);
void asr_stream_destroy(asr_stream* s);

/* Message of the last failure on `e` (or process-wide when e is NULL). */
const char* asr_enc_last_error(const asr_enc* e);

#if defined(__GNUC__)
#pragma GCC visibility pop
#endif
#ifdef __cplusplus
}
#endif
#endif /* ASR_ENC_H */
