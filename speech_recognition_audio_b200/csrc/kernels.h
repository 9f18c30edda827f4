// Host-side declarations of the kernel launchers (one definition each, in
// mel.cu, stem.cu, layer.cu, gemm.cu).
#pragma once

#include <algorithm>
#include <utility>

#include "common.cuh"
#include "gemm.cuh"

namespace asr {

// Launch with programmatic stream serialisation (see pdl_wait in common.cuh).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Tables of the log-mel kernel, built on the device by launch_mel_tables.
constexpr int kMelMaxWeights = 1024;  // taps of any filterbank of <= 128 filters over 201 bins: <= 2 * 201 + 128
struct MelTables {
  float2 w200[200];   // exp(-2 pi i j / 200)
  float2 w400[201];   // exp(-2 pi i k / 400)
  float hann[400];    // periodic Hann
  int fstart[128], fcount[128], foff[128];
  float fw[kMelMaxWeights];  // non-zero filter weights, filter-major (an empty filter has one zero tap)
  // The same taps as (bin | last-tap-of-its-filter << 8 | filter << 9), and
  // their split over the 8 threads of a frame: thread t takes taps
  // [tpart[t], tpart[t+1]), whole filters, about equal counts.
  int tcode[kMelMaxWeights];
  int tpart[9];
};

// One clip of a variable-length batch (log-mel view): samples at pcm + s_off,
// frames = n / 160 at mel + n_mels * f_off ([n_mels][frames]), and the index
// of its first 32-frame group.  `left` samples before pcm + s_off are real
// audio (a streamed window's history): the centred frames read them instead
// of reflecting; 0 for a clip that starts there.
struct MelClip {
  long long s_off, n, f_off;
  int frames, g_off, left;
};
struct MelArgs {
  const float* pcm;
  float* mel;                 // raw log10 mel
  unsigned int* clip_max;     // [batch], order-preserving encoding, zero before the launch
  int n_mels, batch, n_groups;
  long long n_samples;        // uniform batches: samples per clip
  int n_frames;               // uniform batches: frames per clip
  const MelClip* clips;       // variable-length batches: [batch] (device), else null
};
int mel_groups(long long n_frames);  // 32-frame groups of a clip

cudaError_t launch_mel_tables(int n_mels, MelTables* tab, cudaStream_t st);
cudaError_t launch_log_mel(const MelArgs& args, const MelTables* tab, cudaStream_t st);
cudaError_t launch_log_mel(const float* pcm, long long n_samples, int batch, int n_mels, const MelTables* tab,
                           float* mel_raw, unsigned int* clip_max, cudaStream_t st);
cudaError_t launch_mel_normalize(const float* raw, const unsigned int* clip_max, long long per_clip, int batch,
                                 float* out, cudaStream_t st);
cudaError_t launch_mel_normalize_transpose(const float* raw, const unsigned int* clip_max, int batch, int n_mels,
                                           int n_frames, void* out, int kind, cudaStream_t st);

// Variable-length batches.  One conv chunk: its clip, its first frame within
// the clip, its valid frames (chunk_frames except for a clip's last chunk)
// and the packed token row of its first token.
struct ChunkDesc {
  int clip, frame0, nvalid, tok_dst;
};
// Per-clip layout of a variable-length batch, computed on the host.
struct VarClip {
  long long s_off, n, f_off;          // samples: offset, count; frames: offset
  int frames, g_off;                   // frames, first 32-frame mel group
  int left;                            // real samples before s_off (MelClip::left)
  int chunk_off, chunks;               // conv chunks
  int tok_off, tokens;                 // packed token rows
  int win_off, wins;                   // attention windows
};
constexpr int kVarClipsPerLaunch = 32;
struct VarClipBatch {
  int first, count;
  VarClip c[kVarClipsPerLaunch];
};
// Writes the mel descriptors, the chunk descriptors and the window offsets
// of the clips in `vb` (one block per clip); with last != 0 also the final
// window offset cu[n_win] = n_tokens.
cudaError_t launch_varlen_fill(const VarClipBatch& vb, int chunk_frames, int window, int t3, MelClip* mc,
                               ChunkDesc* cd, int* cu, int last, int n_win, int n_tokens, cudaStream_t st);
cudaError_t launch_conv1_im2col_varlen(const float* mel_raw, const unsigned int* clip_max, int n_chunks, int n_mels,
                                       int chunk_frames, int phase, const ChunkDesc* cd, const MelClip* mc, void* a,
                                       int kind, cudaStream_t st);
// layout: 0 [chunk][T][F], 1 parity planes per chunk, 2 packed (S2 rows per
// chunk: conv1 planes [4][chunk][S2][F / 2] at level 1, conv2 [chunk][S2][F]
// at level 2).
cudaError_t launch_mask_short_chunks(void* act, const ChunkDesc* cd, int n_chunks, int chunk_frames, int level, int T,
                                     int F, int C, int layout, int S2, int es, cudaStream_t st);
cudaError_t launch_compact_tokens(const float* xpad, float* x, const ChunkDesc* cd, int n_chunks, int t3, int d,
                                  cudaStream_t st);

// A operand of the first Conv2D (1 -> C, k3 s2 p1) as a GEMM: per output
// position of each chunk of chunk_frames frames, its 9 normalised log-mel
// taps (kh * 3 + kw) as bf16 in a row of 16 (taps 9..15 zero).  Rows
// (phase = layout): 0 [chunks][T1][F1]; 1 (T1, F1 even) the parity planes
// [chunks][t % 2][f % 2][T1 / 2][F1 / 2] read by the phase-mode conv2;
// 2 the packed planes [t % 2][f % 2][chunks][T1 / 2 + 1][F1 / 2], whose last
// row per chunk is zero.
// a: rows of the kind's element type (bf16, f16, or fp32 for KIND_TF32).
cudaError_t launch_conv1_im2col(const float* mel_raw, const unsigned int* clip_max, int batch, int n_mels,
                                int n_frames, int chunk_frames, int phase, void* a, int kind, cudaStream_t st);

// y: bf16 (out_kind KIND_BF16), fp32 (KIND_TF32) or f16 (KIND_F16).
cudaError_t launch_layer_norm(const float* x, const float* g, const float* b, long long M, int D, float eps,
                              void* y, int out_kind, cudaStream_t st);

// tcgen05 attention for segments of at most 128 tokens (attn_tc.cu).
bool make_tmap_qkv(CUtensorMap* map, const void* qkv, long long T, int H);
cudaError_t launch_attention_tc(const CUtensorMap& tm_qkv, const void* qkv, const int* cu, int n_seg, int H, void* out,
                                int* status, unsigned long long limit_ns, bool f16, cudaStream_t st);
// fp32 attention on the CUDA cores (attn_f32.cu): the fp32-weight path.
cudaError_t launch_attention_f32(const float* qkv, const int* cu, int n_seg, int max_seg, int H, float* out,
                                 cudaStream_t st);
// tcgen05 flash attention for segments of any length (attn_fa.cu).
cudaError_t launch_attention_fa(const CUtensorMap& tm_qkv, const int* cu, int n_seg, int max_seg, int H, void* out,
                                int* status, unsigned long long limit_ns, bool f16, cudaStream_t st);

// Audio-embedding splice (splice.cu).  Element types match ASR_DTYPE_*.
enum : int { SPLICE_BF16 = 0, SPLICE_F32 = 1, SPLICE_F16 = 2 };
enum : int { SPLICE_OK = 0, SPLICE_E_ID = 1, SPLICE_E_COUNT = 2 };
cudaError_t launch_splice(const int* ids, long long n_ids, int placeholder, const void* table, int vocab,
                          int table_dtype, const float* frames, long long n_frames, int D, void* out, int out_dtype,
                          int* rank, int* status, int num_sms, cudaStream_t st);

cudaError_t launch_fill_windows(int* cu, int batch, int tokens_per_clip, int window, int n_win_per_clip,
                                cudaStream_t st);
// 16-bit (bf16, or f16 with f16 != 0) to fp32.
cudaError_t launch_bf16_to_f32(const void* in, float* out, long long n, bool f16, cudaStream_t st);
cudaError_t launch_gelu(const float* x, float* y, long long n, cudaStream_t st);
cudaError_t launch_wait_probe(unsigned long long limit_ns, int* status, cudaStream_t st);

// GEMM engine launch (gemm.cu).
constexpr int kGemmSlots = 6;
struct GemmB {              // weight operand [N, K] (bf16, or fp32 for KIND_TF32) + its TMA maps
  const void* ptr = nullptr;
  int N = 0, K = 0;
  int kind = KIND_BF16;
  CUtensorMap map[kGemmSlots];  // box rows 256, 128, 240, 64, 160, 120 (index by gemm_bn_slot)
  CUtensorMap map3;             // 3-D {64, N, K / 64} view, box {64, 128, 2} (16-bit kinds, K % 128 == 0)
  bool has3 = false;
};
// 3-D view {64 elements, rows, cols / 64} of a row-major 16-bit [rows][cols]
// matrix with a box of two 64-element k-blocks of box_rows rows (the A and B
// stages of the CTA-pair kernel's two-k-block pipeline); cols % 128 == 0.
bool make_tmap_3d16(CUtensorMap* map, const void* ptr, unsigned long long rows, unsigned long long cols,
                    unsigned long long row_stride_elems, unsigned int box_rows, int kind);
int gemm_bn_slot(int bn);
bool make_tmap_bf16(CUtensorMap* map, const void* ptr, unsigned long long rows, unsigned long long cols,
                    unsigned long long row_stride_elems, unsigned int box_rows);
// fp32 activation map (box 32 x box_rows: one 128-byte row per box row).
bool make_tmap_f32(CUtensorMap* map, const void* ptr, unsigned long long rows, unsigned long long cols,
                   unsigned long long row_stride_elems, unsigned int box_rows);
// A-operand map of an activation of the kind's element type.
bool make_tmap_act(int kind, CUtensorMap* map, const void* ptr, unsigned long long rows, unsigned long long cols,
                   unsigned long long row_stride_elems, unsigned int box_rows);
bool make_weight_maps(GemmB& w);
// 4-D strided-box map over a conv activation [n_img, T_in, F_in, C] (see ConvBox),
// elements of the kind's type (box inner extent: one 128-byte row).
bool make_tmap_convbox(CUtensorMap* map, const void* ptr, int C, int F_in, int T_in, int n_img, int F_out, int sf,
                       int TR, int st, int kind = KIND_BF16);
// 4-D dense-box map over a parity-plane activation [n_planes][T_h][F_h][C]
// (ConvBox phase mode): box {row elements, F_out, TR, 1}.
bool make_tmap_convphase(CUtensorMap* map, const void* ptr, int C, int F_h, int T_h, int n_planes, int F_out, int TR,
                         int kind = KIND_BF16);
// Picks the tile for an M x N problem on num_sms SMs: a positive width is a
// one-SM 128 x bn tile, a negative one a CTA-pair 256 x |bn| tile.
int gemm_pick_bn(int M, int N, int num_sms, bool gather);
// Tile width for fp32 (tf32) operands: one-SM tiles only.
int gemm_pick_bn_tf32(int M, int N, int num_sms);
// Tile choice for a conv-box GEMM with n_sub 128-row sub-tiles.
int gemm_pick_bn_conv(int n_sub, int N, int num_sms);
// TMA map of a GEMM output [rows, cols] (row stride in elements), box 32 x 32,
// fp32 (128-byte swizzle) or bf16 (64-byte swizzle): the epilogue's store map.
bool make_tmap_out(CUtensorMap* map, const void* ptr, unsigned long long rows, unsigned long long cols,
                   unsigned long long row_stride_elems, bool f32);
// a_map: TMA map of A (box 128 x 64), or null with p.g set for the implicit-GEMM mode.
// out_map: store map of the output (make_tmap_out), or null for plain stores;
// ignored for the position and SwiGLU epilogues.
// a_map3: 3-D map of A (make_tmap_3d16, box rows 128) or null; with it, plain
// 256-wide CTA-pair launches run two k-blocks per pipeline stage.
// epi = EPI_RESID | EPI_LN (16-bit kinds; needs a_map3 and p.ln_* set,
// p.ldo % 8 == 0): the residual update and the LayerNorm of the updated
// rows into p.ln_h; the launch runs whole 256 x 256 pair tiles (bn and
// out_map ignored).  cudaErrorInvalidValue when the shape does not allow it.
cudaError_t launch_gemm(const CUtensorMap* a_map, const GemmB& w, GemmParams p, int epi, int bn, int num_sms,
                        cudaStream_t st, const CUtensorMap* out_map, const CUtensorMap* a_map3 = nullptr);
// Whether launch_gemm takes EPI_RESID | EPI_LN for this weight (16-bit
// kind, K % 128 == 0, N % 32 == 0, enough resident CTA pairs).
bool gemm_ln_supported(const GemmB& w, int num_sms);

}  // namespace asr
