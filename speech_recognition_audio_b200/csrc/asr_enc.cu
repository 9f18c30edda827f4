// C ABI of the encoder library: geometry queries, weight repacking, the
// workspace plan and the forward launch sequence.
//
// Forward of one batch (conv2d stem; "MOSS-Transcribe-preview-2B-GGUF",
// Architecture table):
//   log-mel -> conv1 (CUDA cores) -> conv2, conv3 (implicit GEMM, bias+GELU)
//   -> conv_out (+ per-chunk sinusoidal positions) -> 32 x [LN1 -> QKV ->
//   windowed attention -> out-proj + residual -> LN2 -> fc1 + GELU -> fc2 +
//   residual] -> ln_post -> proj1 + GELU -> proj2 -> gate/up + SwiGLU -> down.
// Conv1D stem (whisper-small geometry, "CrisperWhisper -> ONNX", What this
// exports instead / Results): log-mel -> transpose -> conv1 (k3 s1) + GELU ->
// conv2 (k3 s2) + GELU + global positions -> 12 layers with full attention
// -> final LayerNorm.
#include <climits>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/asr_enc.h"
#include "../../include/asr_ops.h"
#include "kernels.h"

using namespace asr;

namespace {

std::mutex g_err_mu;
std::string g_err = "";

constexpr unsigned long long kWaitLimitNs = 2000ull * 1000 * 1000;  // 2 s per device wait

struct LayerW {
  GemmB qkv, o, fc1, fc2;
  float *bqkv, *bo, *b1, *b2, *ln1g, *ln1b, *ln2g, *ln2b;
};

struct ActMaps {
  const void* ws = nullptr;
  int64_t n = 0, T = 0, chunks = 0;
  int batch = 0;
  unsigned taps = 0;
  CUtensorMap h, att, ff, c3, p1, p2, gu;
  CUtensorMap a1;          // conv1 taps [positions, 16] (box 128 x 64: columns 16..63 read as zeros)
  CUtensorMap cin2, cin3;  // conv-box A maps of the two stem GEMMs
  CUtensorMap qkv;         // 128-row boxes of the QKV buffer (tcgen05 attention)
  // Store maps of the GEMM outputs (32 x 32 boxes): residual stream, QKV,
  // FFN hidden, head, adapter hidden, conv outputs.
  CUtensorMap o_x, o_qkv, o_ff, o_p1, o_p2, o_c2, o_c3, o_c1;
  // QKV split (16-bit, T not a multiple of 256): rows [0, qkv_main) on
  // CTA-pair tiles, the last T - qkv_main on one-SM tiles (A and output maps
  // of those rows), concurrently on the encoder's side stream
  int64_t qkv_main = 0;
  CUtensorMap h_tail, o_qkv_tail;
  // 3-D companions of the plain activation maps (boxes of 128 rows x two
  // 64-column k-blocks, 16-bit kinds with K a multiple of 128): with one, the
  // CTA-pair GEMM loads two k-blocks of A per TMA copy.
  static constexpr int kMax3 = 8;
  const CUtensorMap* src3[kMax3] = {};
  CUtensorMap map3[kMax3];
  int n3 = 0;
  bool add3(const CUtensorMap* m2, const void* ptr, unsigned long long rows, unsigned long long cols, int kind) {
    if (n3 >= kMax3) return false;
    if (kind == KIND_TF32 || cols % 128) return true;  // no companion: the 2-D path
    if (!make_tmap_3d16(&map3[n3], ptr, rows, cols, cols, 128, kind)) return false;
    src3[n3++] = m2;
    return true;
  }
  const CUtensorMap* companion3(const CUtensorMap* m2) const {
    for (int i = 0; i < n3; ++i)
      if (src3[i] == m2) return &map3[i];
    return nullptr;
  }
};

struct Plan {
  int64_t n = 0, Tc = 0, T = 0;
  int B = 0, F = 0, nwin_clip = 0, nwin = 0, max_win = 0, chunks = 0;
  int T1 = 0, F1 = 0, T2 = 0, F2 = 0, T3 = 0, F3 = 0;
  // conv1 / conv2 output rows (positions) and, in the packed layout, the
  // per-chunk row stride S2 = T2 + 1 of the conv1 planes and of conv2's output
  int S2 = 0;
  int64_t rows1 = 0, rows2 = 0;
  // Variable-length batches (conv2d stem): per-clip layout, padded conv_out
  // rows (every chunk padded to T3 tokens), total frames and mel groups.
  bool varlen = false, has_short = false;
  std::vector<VarClip> clips;
  int64_t Tpad = 0, n_total = 0, Ftot = 0;
  int n_groups = 0;
  size_t off_clipmax = 0, off_cu = 0, off_mel = 0, off_a1 = 0, off_c1 = 0, off_c2 = 0, off_c3 = 0, off_melT = 0, off_x = 0,
         off_h = 0, off_qkv = 0, off_att = 0, off_ff = 0, off_p1 = 0, off_p2 = 0, off_gu = 0, off_pcm = 0, off_out = 0,
         off_mclips = 0, off_chunkd = 0, off_xpad = 0, off_skflags = 0, off_lncnt = 0, off_lnpart = 0;
  size_t off_tap[ASR_TAP_COUNT] = {0, 0, 0, 0, 0};
  size_t tap_bytes[ASR_TAP_COUNT] = {0, 0, 0, 0, 0};
  size_t total = 0;
};

int64_t conv_len(int64_t n, int k, int s, int p) { return (n + 2 * p - k) / s + 1; }

bool geom_valid(const asr_geometry* g, std::string* why) {
  auto fail = [&](const char* m) {
    if (why) *why = m;
    return false;
  };
  if (!g) return fail("geometry is NULL");
  if (g->stem != ASR_STEM_CONV2D_CHUNKED && g->stem != ASR_STEM_CONV1D) return fail("unknown stem");
  if (g->n_mels <= 0 || g->n_mels > 128) return fail("n_mels must be 1..128");
  if (g->n_fft != 400 || g->hop != 160) return fail("only n_fft 400 / hop 160 are implemented");
  if (g->stem == ASR_STEM_CONV2D_CHUNKED) {
    if (g->chunk_frames <= 0) return fail("chunk_frames must be > 0");
    if (g->conv_ch <= 0 || g->conv_ch % 8 || g->conv_ch > 512) return fail("conv_ch must be a multiple of 8, <= 512");
  }
  if (g->d_model <= 0 || g->d_model % 128 || g->d_model > 2048) return fail("d_model must be a multiple of 128, <= 2048");
  if (g->head_dim != 64 || g->n_heads * g->head_dim != g->d_model) return fail("head_dim must be 64 and n_heads*64 == d_model");
  if (g->d_ffn <= 0 || g->d_ffn % 64) return fail("d_ffn must be a positive multiple of 64");
  if (g->n_layers < 0) return fail("n_layers < 0");
  if (g->window_tokens < 0) return fail("window_tokens < 0");
  if (g->pos_mode != ASR_POS_PER_CHUNK && g->pos_mode != ASR_POS_GLOBAL) return fail("unknown pos_mode");
  if (g->pos_mode == ASR_POS_PER_CHUNK && g->stem != ASR_STEM_CONV2D_CHUNKED) return fail("per-chunk positions need the chunked stem");
  if ((g->proj1_out == 0) != (g->proj2_out == 0)) return fail("proj1_out and proj2_out must both be set or both 0");
  if (g->proj1_out && (g->proj1_out % 64 || g->proj2_out % 128 || g->proj2_out > 2048)) return fail("head widths: proj1 % 64, proj2 % 128, <= 2048");
  if ((g->adapter_hidden == 0) != (g->adapter_out == 0)) return fail("adapter_hidden and adapter_out must both be set or both 0");
  if (g->adapter_hidden && (g->adapter_hidden % 16 || g->adapter_out % 16)) return fail("adapter widths must be multiples of 16");
  if (g->adapter_hidden && !g->proj1_out) return fail("the adapter needs the head projections");
  if (!(g->ln_eps > 0.f)) return fail("ln_eps must be > 0");
  if (g->dtype != ASR_DTYPE_BF16 && g->dtype != ASR_DTYPE_F32 && g->dtype != ASR_DTYPE_F16) return fail("unknown dtype");
  return true;
}

int d_out(const asr_geometry* g) {
  if (g->adapter_hidden) return g->adapter_out;
  if (g->proj2_out) return g->proj2_out;
  return g->d_model;
}

struct WSpec {
  std::string name;
  int ndim;
  int64_t shape[4];
};

std::vector<WSpec> weight_specs(const asr_geometry* g) {
  std::vector<WSpec> s;
  const int64_t d = g->d_model, C = g->conv_ch;
  auto add = [&](const std::string& n, std::initializer_list<int64_t> sh) {
    WSpec w;
    w.name = n;
    w.ndim = static_cast<int>(sh.size());
    int i = 0;
    for (int64_t v : sh) w.shape[i++] = v;
    for (; i < 4; ++i) w.shape[i] = 1;
    s.push_back(w);
  };
  if (g->stem == ASR_STEM_CONV2D_CHUNKED) {
    const int64_t f3 = conv_len(conv_len(conv_len(g->n_mels, 3, 2, 1), 3, 2, 1), 3, 2, 1);
    add("conv1.w", {C, 1, 3, 3}); add("conv1.b", {C});
    add("conv2.w", {C, C, 3, 3}); add("conv2.b", {C});
    add("conv3.w", {C, C, 3, 3}); add("conv3.b", {C});
    add("conv_out.w", {d, C * f3});
  } else {
    add("conv1.w", {d, g->n_mels, 3}); add("conv1.b", {d});
    add("conv2.w", {d, d, 3}); add("conv2.b", {d});
  }
  for (int l = 0; l < g->n_layers; ++l) {
    const std::string p = "layers." + std::to_string(l) + ".";
    add(p + "ln1.g", {d}); add(p + "ln1.b", {d});
    add(p + "q.w", {d, d}); add(p + "q.b", {d});
    add(p + "k.w", {d, d}); add(p + "k.b", {d});
    add(p + "v.w", {d, d}); add(p + "v.b", {d});
    add(p + "o.w", {d, d}); add(p + "o.b", {d});
    add(p + "ln2.g", {d}); add(p + "ln2.b", {d});
    add(p + "fc1.w", {g->d_ffn, d}); add(p + "fc1.b", {g->d_ffn});
    add(p + "fc2.w", {d, g->d_ffn}); add(p + "fc2.b", {d});
  }
  add("ln_post.g", {d}); add("ln_post.b", {d});
  if (g->proj1_out) {
    add("proj1.w", {g->proj1_out, d}); add("proj1.b", {g->proj1_out});
    add("proj2.w", {g->proj2_out, g->proj1_out}); add("proj2.b", {g->proj2_out});
  }
  if (g->adapter_hidden) {
    add("adapter.gate.w", {g->adapter_hidden, g->proj2_out});
    add("adapter.up.w", {g->adapter_hidden, g->proj2_out});
    add("adapter.down.w", {g->adapter_out, g->adapter_hidden});
  }
  return s;
}

int64_t numel(const WSpec& w) {
  int64_t n = 1;
  for (int i = 0; i < w.ndim; ++i) n *= w.shape[i];
  return n;
}

// Tokens of a chunk of L frames after three k3 s2 p1 convolutions.
int64_t chunk_tokens(int64_t L) { return conv_len(conv_len(conv_len(L, 3, 2, 1), 3, 2, 1), 3, 2, 1); }

// Stream-K flags of the residual GEMMs (one per CTA-pair slot, CTA and
// epilogue warp); zeroed at the start of every forward, each cleared again by
// the tile owner that consumed it.
size_t sk_flags_bytes(const asr_enc* e);
size_t ln_count_bytes(int64_t T);
int ln_parts(const asr_enc* e);

// Output rows of conv1 and conv2 (conv2d stem): [chunk][T][F] each, or in the
// packed layout the four conv1 parity planes [plane][chunk][S2][F1 / 2] and
// conv2's [chunk][S2][F2], S2 = T2 + 1 (one zero row per chunk).
void set_stem_rows(bool packed, Plan* p) {
  p->S2 = packed ? p->T2 + 1 : 0;
  p->rows1 = packed ? 4LL * p->chunks * p->S2 * (p->F1 / 2) : (int64_t)p->chunks * p->T1 * p->F1;
  p->rows2 = (int64_t)p->chunks * (packed ? p->S2 : p->T2) * p->F2;
}

// Tokens per clip, or -1.  frames = floor(n / hop) (the trailing STFT frame
// dropped); the conv2d stem's last chunk may be short.
int64_t tokens_from_frames(const asr_geometry* g, int64_t frames) {
  if (frames <= 0) return -1;
  if (g->stem == ASR_STEM_CONV2D_CHUNKED) {
    const int64_t full = frames / g->chunk_frames, rest = frames % g->chunk_frames;
    return full * chunk_tokens(g->chunk_frames) + (rest ? chunk_tokens(rest) : 0);
  }
  return conv_len(conv_len(frames, 3, 1, 1), 3, 2, 1);
}

int64_t tokens_per_clip(const asr_geometry* g, int64_t n) {
  if (!geom_valid(g, nullptr) || n <= g->n_fft / 2) return -1;
  const int64_t frames = n / g->hop;
  if (g->stem == ASR_STEM_CONV2D_CHUNKED) {
    const int64_t full = frames / g->chunk_frames, rest = frames % g->chunk_frames;
    return full * chunk_tokens(g->chunk_frames) + (rest ? chunk_tokens(rest) : 0);
  }
  return conv_len(conv_len(frames, 3, 1, 1), 3, 2, 1);
}

// A batch the uniform plan handles: whole hops, and for the conv2d stem
// whole chunks (a short last chunk goes through the variable-length plan).
bool uniform_ok(const asr_geometry* g, int64_t n) {
  if (n % g->hop) return false;
  return g->stem != ASR_STEM_CONV2D_CHUNKED || (n / g->hop) % g->chunk_frames == 0;
}

// Sinusoidal positions [rows, d]: d/2 frequencies exp(-ln(1e4) i / (d/2 - 1)),
// [sin(p w_i) | cos(p w_i)].
std::vector<float> build_pe(int rows, int d) {
  std::vector<float> pe((size_t)rows * d);
  const int half = d / 2;
  const double inc = log(10000.0) / (half - 1);
  for (int p = 0; p < rows; ++p)
    for (int i = 0; i < half; ++i) {
      const double a = p * exp(-inc * i);
      pe[(size_t)p * d + i] = (float)sin(a);
      pe[(size_t)p * d + half + i] = (float)cos(a);
    }
  return pe;
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace

struct asr_enc {
  asr_geometry g;
  // Operand kind of every GEMM and element size of the activations between
  // them: bf16 (bf16 weights), or fp32 with tf32 MMAs (fp32 weights).
  int kind = KIND_BF16;
  int es = 2;
  asr_alloc_fn alloc = nullptr;
  asr_free_fn free_fn = nullptr;
  void* ctx = nullptr;
  int device = 0, num_sms = 148;
  void* slab = nullptr;
  size_t slab_bytes = 0, slab_used = 0;
  std::string err;
  // stem
  float *c1b = nullptr, *c2b = nullptr, *c3b = nullptr;
  GemmB c1, c2, c3, cout;  // conv stem GEMMs (conv1: [C][16] taps kh*3+kw, 9..15 zero)
  bool box2 = false, box3 = false;  // conv GEMMs read A as strided TMA boxes (else cp.async gather)
  bool phase2 = false;              // conv1 writes parity planes, conv2 reads dense boxes
  // Packed stem layout (parity planes, odd conv2 length per chunk): the
  // chunks follow each other along time with one zero row after each (conv1
  // planes and conv2 output alike), so the stride-2 convolutions read the
  // neighbour chunk's zero row as their padding and conv2 / conv3 tiles run
  // across chunk boundaries (no partly empty tiles).
  bool packed = false;
  // fc2 of every block also writes the next LayerNorm's output (EPI_LN):
  // possible for 16-bit weights of suitable shape (ln_fuse), used when
  // asr_enc_set_ln_fusion turned it on (off by default: with the single-wave
  // LayerNorm kernel the separate launches are faster).
  bool ln_fuse = false, ln_fuse_on = false;
  float* pe = nullptr;
  int pe_rows = 0;
  std::vector<LayerW> layers;
  float *lnpg = nullptr, *lnpb = nullptr, *bp1 = nullptr, *bp2 = nullptr;
  GemmB p1, p2, gu, down;
  MelTables* mel_tab = nullptr;
  int* status = nullptr;
  unsigned taps = 0;
  cudaStream_t last_stream = nullptr;
  // The last uniform forward recorded as a CUDA graph (keyed on its
  // pointers and shape) and replayed while the key matches: one launch
  // instead of ~240, programmatic (PDL) edges kept.  `graphs` off after a
  // failed capture or by asr_enc_set_graphs.
  struct GraphKey {
    const float* pcm = nullptr;
    float* out = nullptr;
    void* ws = nullptr;
    int64_t n = 0;
    int B = 0;
    unsigned taps = 0;
    bool operator==(const GraphKey& o) const {
      return pcm == o.pcm && out == o.out && ws == o.ws && n == o.n && B == o.B && taps == o.taps;
    }
  } gkey;
  cudaGraphExec_t gexec = nullptr;
  int glaunches = 0;
  cudaStream_t cap_st = nullptr;
  // side stream and fork / join events of the split QKV projection
  cudaStream_t aux_st = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
  bool graphs = true;
  bool have_last = false;
  Plan last_plan;
  void* last_ws = nullptr;
  ActMaps maps;
  // kernel timing
  bool prof = false;
  std::vector<cudaEvent_t> ev_pool;
  size_t ev_used = 0;
  std::vector<std::pair<int, size_t>> prof_recs;  // (stage class, index of the first of two events)
  int launches = 0;
};

namespace {

asr_status fail(asr_enc* e, asr_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  if (e) e->err = buf;
  std::lock_guard<std::mutex> lk(g_err_mu);
  g_err = buf;
  return st;
}

#define ASR_CUDA(e, call)                                                                                   \
  do {                                                                                                      \
    cudaError_t _r = (call);                                                                                \
    if (_r != cudaSuccess) return fail((e), ASR_E_CUDA, "%s failed: %s", #call, cudaGetErrorString(_r));   \
  } while (0)

void* slab_take(asr_enc* e, size_t bytes) {
  const size_t off = align_up(e->slab_used, 1024);
  if (off + bytes > e->slab_bytes) return nullptr;
  e->slab_used = off + bytes;
  return static_cast<char*>(e->slab) + off;
}

float bf16_to_float(uint16_t h) {
  const uint32_t u = static_cast<uint32_t>(h) << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

// IEEE binary16 -> float (exact: every half is a float).
float f16_to_float(uint16_t h) {
  const uint32_t sign = static_cast<uint32_t>(h >> 15) << 31;
  const int ex = (h >> 10) & 31;
  const uint32_t man = h & 1023;
  float f;
  if (ex == 0) {
    f = std::ldexp(static_cast<float>(man), -24);  // zero or subnormal
  } else if (ex == 31) {
    const uint32_t u = 0x7F800000u | (man << 13);  // inf or nan
    memcpy(&f, &u, 4);
  } else {
    const uint32_t u = (static_cast<uint32_t>(ex - 15 + 127) << 23) | (man << 13);
    memcpy(&f, &u, 4);
  }
  if (sign) f = -f;
  return f;
}

// float -> IEEE binary16, round to nearest even (values here are weights:
// finite; overflow saturates to infinity as the rounding rule gives).
uint16_t float_to_f16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  const uint16_t sign = static_cast<uint16_t>((u >> 16) & 0x8000u);
  const float a = std::fabs(f);
  if (!(a == a)) return static_cast<uint16_t>(sign | 0x7E00u);
  if (a >= 65520.0f) return static_cast<uint16_t>(sign | 0x7C00u);
  if (a < 6.103515625e-05f) {  // subnormal range: multiples of 2^-24
    const float q = std::nearbyint(std::ldexp(a, 24));  // default rounding: nearest even
    return static_cast<uint16_t>(sign | static_cast<uint16_t>(q));
  }
  int ex;
  const float m = std::frexp(a, &ex);                        // a = m 2^ex, m in [0.5, 1)
  float q = std::nearbyint(std::ldexp(m, 11));                // 11 significant bits
  if (q >= 2048.0f) {
    q = 1024.0f;
    ++ex;
  }
  const uint32_t bits = (static_cast<uint32_t>(ex - 1 + 15) << 10) | (static_cast<uint32_t>(q) - 1024u);
  return static_cast<uint16_t>(sign | bits);
}

// Copies a weight tensor to the host as float; false if the copy failed.
bool fetch(const void* dptr, int64_t n, int dtype, std::vector<float>* out, cudaError_t* err) {
  out->assign((size_t)n, 0.0f);
  if (dtype == ASR_DTYPE_F32) {
    *err = cudaMemcpy(out->data(), dptr, n * 4, cudaMemcpyDeviceToHost);
    return *err == cudaSuccess;
  }
  std::vector<uint16_t> tmp((size_t)n);
  *err = cudaMemcpy(tmp.data(), dptr, n * 2, cudaMemcpyDeviceToHost);
  if (*err != cudaSuccess) return false;
  for (int64_t i = 0; i < n; ++i) (*out)[i] = dtype == ASR_DTYPE_F16 ? f16_to_float(tmp[i]) : bf16_to_float(tmp[i]);
  return true;
}

uint16_t f2bf(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u) return static_cast<uint16_t>((u >> 16) | ((u & 0xFFFF) ? 0x40 : 0));
  const uint32_t rounding = 0x7FFFu + ((u >> 16) & 1u);
  return static_cast<uint16_t>((u + rounding) >> 16);
}

}  // namespace

// ====================================================================== ABI

extern "C" {

int asr_enc_weight_count(const asr_geometry* g) {
  if (!geom_valid(g, nullptr)) return -1;
  return static_cast<int>(weight_specs(g).size());
}

asr_status asr_enc_weight_info(const asr_geometry* g, int i, const char** name, int* ndim, int64_t shape[4]) {
  std::string why;
  if (!geom_valid(g, &why)) return fail(nullptr, ASR_E_INVAL, "invalid geometry: %s", why.c_str());
  static std::mutex mu;
  static std::map<std::string, std::string> names;  // interned names
  auto s = weight_specs(g);
  if (i < 0 || i >= (int)s.size()) return fail(nullptr, ASR_E_INVAL, "weight index %d out of range", i);
  if (name) {
    std::lock_guard<std::mutex> lk(mu);
    auto it = names.emplace(s[i].name, s[i].name).first;
    *name = it->second.c_str();
  }
  if (ndim) *ndim = s[i].ndim;
  if (shape)
    for (int k = 0; k < 4; ++k) shape[k] = s[i].shape[k];
  return ASR_OK;
}

int64_t asr_enc_tokens(const asr_geometry* g, int64_t n_samples) { return tokens_per_clip(g, n_samples); }

asr_status asr_enc_windows(const asr_geometry* g, int64_t n_samples, int batch, int32_t* cu, int* n) {
  if (!n) return fail(nullptr, ASR_E_INVAL, "n is NULL");
  const int64_t t = tokens_per_clip(g, n_samples);
  if (t < 0 || batch <= 0) return fail(nullptr, ASR_E_INVAL, "invalid geometry, n_samples or batch");
  const int64_t w = g->window_tokens ? g->window_tokens : t;
  const int64_t per = (t + w - 1) / w;
  const int64_t count = per * batch;
  if (count > 0x7FFFFFFF || t * batch > 0x7FFFFFFF) return fail(nullptr, ASR_E_UNSUPPORTED, "partition too large");
  if (cu) {
    if (*n < count + 1) return fail(nullptr, ASR_E_INVAL, "cu capacity %d < %lld", *n, (long long)(count + 1));
    int idx = 0;
    cu[idx++] = 0;
    for (int b = 0; b < batch; ++b)
      for (int64_t j = 0; j < per; ++j) cu[idx++] = static_cast<int32_t>(b * t + std::min((j + 1) * w, t));
  }
  *n = static_cast<int>(count);
  return ASR_OK;
}

const char* asr_enc_last_error(const asr_enc* e) {
  if (e) return e->err.c_str();
  std::lock_guard<std::mutex> lk(g_err_mu);
  static thread_local std::string copy;
  copy = g_err;
  return copy.c_str();
}

void asr_enc_destroy(asr_enc* e) {
  if (!e) return;
  if (e->gexec) cudaGraphExecDestroy(e->gexec);
  if (e->cap_st) cudaStreamDestroy(e->cap_st);
  if (e->aux_st) cudaStreamDestroy(e->aux_st);
  if (e->ev_fork) cudaEventDestroy(e->ev_fork);
  if (e->ev_join) cudaEventDestroy(e->ev_join);
  for (cudaEvent_t ev : e->ev_pool) cudaEventDestroy(ev);
  if (e->slab) {
    if (e->free_fn)
      e->free_fn(e->ctx, e->slab);
    else if (!e->alloc)
      cudaFree(e->slab);
  }
  delete e;
}

asr_status asr_enc_create(const asr_geometry* g, const void* const* weights, int n_weights, asr_alloc_fn alloc,
                          asr_free_fn free_fn, void* alloc_ctx, void* stream, asr_enc** out) {
  if (!out) return fail(nullptr, ASR_E_INVAL, "out is NULL");
  *out = nullptr;
  std::string why;
  if (!geom_valid(g, &why)) return fail(nullptr, ASR_E_UNSUPPORTED, "geometry not supported: %s", why.c_str());
  auto specs = weight_specs(g);
  if (!weights || n_weights != (int)specs.size())
    return fail(nullptr, ASR_E_INVAL, "expected %d weight pointers, got %d", (int)specs.size(), n_weights);
  for (int i = 0; i < n_weights; ++i)
    if (!weights[i]) return fail(nullptr, ASR_E_INVAL, "weight %d (%s) is NULL", i, specs[i].name.c_str());

  asr_enc* e = new asr_enc();
  e->g = *g;
  e->alloc = alloc;
  e->free_fn = free_fn;
  e->ctx = alloc_ctx;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto bad = [&](asr_status s) {
    std::string m = e->err;
    asr_enc_destroy(e);
    fail(nullptr, s, "%s", m.c_str());
    return s;
  };
  if (cudaGetDevice(&e->device) != cudaSuccess) return bad(fail(e, ASR_E_CUDA, "cudaGetDevice failed"));
  if (cudaDeviceGetAttribute(&e->num_sms, cudaDevAttrMultiProcessorCount, e->device) != cudaSuccess)
    return bad(fail(e, ASR_E_CUDA, "cudaDeviceGetAttribute failed"));
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, e->device) != cudaSuccess)
    return bad(fail(e, ASR_E_CUDA, "cudaDeviceGetAttribute failed"));
  if (major != 10) return bad(fail(e, ASR_E_UNSUPPORTED, "this library runs on sm_100 (B200) only; device has sm_%d", major * 10));

  e->kind = g->dtype == ASR_DTYPE_F32 ? KIND_TF32 : g->dtype == ASR_DTYPE_F16 ? KIND_F16 : KIND_BF16;
  e->es = e->kind == KIND_TF32 ? 4 : 2;
  const int rowe = kind_row_elems(e->kind);  // channels per 128-byte row of a conv operand
  const int d = g->d_model, C = g->conv_ch, L = g->n_layers;
  // ---- slab size
  size_t need = 0;
  auto acc = [&](size_t bytes) { need = align_up(need, 1024) + bytes; };
  for (auto& w : specs) acc((size_t)numel(w) * 4);  // generous: every tensor at 4 bytes/element
  // conv kernels are repacked with their input channels padded to a whole
  // 128-byte row per tap (up to 63 extra channels), at up to 4 bytes each
  if (g->stem == ASR_STEM_CONV2D_CHUNKED) {
    acc((size_t)C * 9 * 64 * 4);
    acc((size_t)C * 9 * 64 * 4);
  } else {
    acc((size_t)d * 3 * 64 * 4);
    acc((size_t)d * 3 * 64 * 4);
  }
  const int pe_rows = g->stem == ASR_STEM_CONV2D_CHUNKED
                          ? (int)conv_len(conv_len(conv_len(g->chunk_frames, 3, 2, 1), 3, 2, 1), 3, 2, 1)
                          : 1500;
  acc((size_t)pe_rows * d * 4);
  acc(sizeof(MelTables));
  acc(256);  // status
  e->slab_bytes = align_up(need, 1024) + 4096;
  e->slab = alloc ? alloc(alloc_ctx, e->slab_bytes) : nullptr;
  if (!alloc && cudaMalloc(&e->slab, e->slab_bytes) != cudaSuccess) e->slab = nullptr;
  if (!e->slab) return bad(fail(e, ASR_E_NOMEM, "allocation of %zu bytes failed", e->slab_bytes));

  // The first failing runtime call of the repack is kept and reported.
  cudaError_t cerr = cudaSuccess;
  std::string cwhat;
  auto note = [&](cudaError_t r, const std::string& what) {
    if (r != cudaSuccess && cerr == cudaSuccess) {
      cerr = r;
      cwhat = what;
    }
  };
  auto cuda_fail = [&](const char* what) {
    if (cerr != cudaSuccess) return bad(fail(e, ASR_E_CUDA, "%s failed: %s", cwhat.c_str(), cudaGetErrorString(cerr)));
    return bad(fail(e, ASR_E_CUDA, "%s", what));
  };
  auto up_f32 = [&](const std::vector<float>& v) -> float* {
    float* p = static_cast<float*>(slab_take(e, v.size() * 4));
    if (p) note(cudaMemcpy(p, v.data(), v.size() * 4, cudaMemcpyHostToDevice), "cudaMemcpy (fp32 upload)");
    return p;
  };
  auto up_bf16 = [&](const std::vector<float>& v) -> bf16* {
    std::vector<uint16_t> h(v.size());
    for (size_t i = 0; i < v.size(); ++i) h[i] = f2bf(v[i]);
    bf16* p = static_cast<bf16*>(slab_take(e, h.size() * 2));
    if (p) note(cudaMemcpy(p, h.data(), h.size() * 2, cudaMemcpyHostToDevice), "cudaMemcpy (bf16 upload)");
    return p;
  };
  int wi = 0;
  auto next = [&]() {
    const WSpec& s = specs[wi];
    std::vector<float> v;
    cudaError_t r = cudaSuccess;
    if (!fetch(weights[wi], numel(s), g->dtype, &v, &r)) note(r, "cudaMemcpy of weight " + s.name);
    ++wi;
    return v;
  };
  auto up_f16 = [&](const std::vector<float>& v) -> void* {
    std::vector<uint16_t> h(v.size());
    for (size_t i = 0; i < v.size(); ++i) h[i] = float_to_f16(v[i]);
    void* p = slab_take(e, h.size() * 2);
    if (p) note(cudaMemcpy(p, h.data(), h.size() * 2, cudaMemcpyHostToDevice), "cudaMemcpy (f16 upload)");
    return p;
  };
  auto gemm_w = [&](GemmB& gb, const std::vector<float>& v, int N, int K) -> bool {
    gb.kind = e->kind;
    if (e->kind == KIND_TF32)
      gb.ptr = up_f32(v);  // fp32 weights stay fp32
    else if (e->kind == KIND_F16)
      gb.ptr = up_f16(v);  // f16 weights stay f16 (exact round trip)
    else
      gb.ptr = up_bf16(v);
    gb.N = N;
    gb.K = K;
    return cerr == cudaSuccess && gb.ptr && make_weight_maps(gb);
  };
  note(cudaStreamSynchronize(st), "cudaStreamSynchronize");
  if (g->stem == ASR_STEM_CONV2D_CHUNKED) {
    const int f3 = (int)conv_len(conv_len(conv_len(g->n_mels, 3, 2, 1), 3, 2, 1), 3, 2, 1);
    auto w1 = next();  // [C][kh*3+kw] -> rows of 16
    std::vector<float> r1((size_t)C * 16, 0.0f);
    for (int o = 0; o < C; ++o)
      for (int k = 0; k < 9; ++k) r1[(size_t)o * 16 + k] = w1[(size_t)o * 9 + k];
    if (!gemm_w(e->c1, r1, C, 16)) return cuda_fail("conv1 weight upload / TMA map failed");
    e->c1b = up_f32(next());
    // Conv-box mode needs F_out | 128 (a 128-row tile = whole output rows);
    // fp32 operands have no gather fallback.
    const int f1 = (int)conv_len(g->n_mels, 3, 2, 1), f2 = (int)conv_len(f1, 3, 2, 1);
    e->box2 = f2 > 0 && 128 % f2 == 0 && (128 / f2) * 2 <= 256 && f2 * 2 <= 256;
    e->box3 = f3 > 0 && 128 % f3 == 0 && (128 / f3) * 2 <= 256 && f3 * 2 <= 256;
    const int t1 = (int)conv_len(g->chunk_frames, 3, 2, 1);
    e->phase2 = e->box2 && t1 % 2 == 0 && f1 % 2 == 0 && f2 == f1 / 2;
    const int t2 = (int)conv_len(t1, 3, 2, 1);
    e->packed = e->phase2 && e->box3 && t2 % 2 == 1;
    if (e->kind == KIND_TF32 && !(e->box2 && e->box3))
      return bad(fail(e, ASR_E_UNSUPPORTED, "fp32 weights need conv outputs whose frequency rows divide 128"));
    for (int layer = 0; layer < 2; ++layer) {
      // [o][c][kh][kw] -> [o][tap = kw*3+kh][c], channels padded to 64 per tap in box mode
      auto w = next();
      const bool box = layer == 0 ? e->box2 : e->box3;
      const int cp = box ? (C + rowe - 1) / rowe * rowe : C;
      std::vector<float> r((size_t)C * 9 * cp, 0.0f);
      for (int o = 0; o < C; ++o)
        for (int c = 0; c < C; ++c)
          for (int kh = 0; kh < 3; ++kh)
            for (int kw = 0; kw < 3; ++kw)
              r[(size_t)o * 9 * cp + (kw * 3 + kh) * cp + c] = w[(((size_t)o * C + c) * 3 + kh) * 3 + kw];
      if (!gemm_w(layer == 0 ? e->c2 : e->c3, r, C, 9 * cp)) return cuda_fail("conv weight upload / TMA map failed");
      auto b = next();
      (layer == 0 ? e->c2b : e->c3b) = up_f32(b);
    }
    auto wo = next();  // [d][c*f3 + f] -> [d][f*C + c]
    std::vector<float> r((size_t)d * C * f3);
    for (int o = 0; o < d; ++o)
      for (int c = 0; c < C; ++c)
        for (int f = 0; f < f3; ++f) r[(size_t)o * C * f3 + f * C + c] = wo[(size_t)o * C * f3 + c * f3 + f];
    if (!gemm_w(e->cout, r, d, C * f3)) return cuda_fail("conv_out upload / TMA map failed");
  } else {
    // Conv1D stem: always conv-box mode (F_out = 1, 128 output frames per tile).
    e->box2 = e->box3 = true;
    const int M = g->n_mels;
    const int mp = (M + rowe - 1) / rowe * rowe, dp = (d + rowe - 1) / rowe * rowe;
    auto w1 = next();  // [d][c][k] -> [d][k][c] with channels padded to 64
    std::vector<float> r1((size_t)d * 3 * mp, 0.0f);
    for (int o = 0; o < d; ++o)
      for (int c = 0; c < M; ++c)
        for (int k = 0; k < 3; ++k) r1[(size_t)o * 3 * mp + k * mp + c] = w1[((size_t)o * M + c) * 3 + k];
    if (!gemm_w(e->c2, r1, d, 3 * mp)) return cuda_fail("conv1 upload failed");
    e->c2b = up_f32(next());
    auto w2 = next();
    std::vector<float> r2((size_t)d * 3 * dp, 0.0f);
    for (int o = 0; o < d; ++o)
      for (int c = 0; c < d; ++c)
        for (int k = 0; k < 3; ++k) r2[(size_t)o * 3 * dp + k * dp + c] = w2[((size_t)o * d + c) * 3 + k];
    if (!gemm_w(e->c3, r2, d, 3 * dp)) return cuda_fail("conv2 upload failed");
    e->c3b = up_f32(next());
  }
  e->layers.resize(L);
  for (int l = 0; l < L; ++l) {
    LayerW& lw = e->layers[l];
    lw.ln1g = up_f32(next());
    lw.ln1b = up_f32(next());
    std::vector<float> wqkv, bqkv;
    for (int j = 0; j < 3; ++j) {
      auto w = next();
      auto b = next();
      wqkv.insert(wqkv.end(), w.begin(), w.end());
      bqkv.insert(bqkv.end(), b.begin(), b.end());
    }
    if (!gemm_w(lw.qkv, wqkv, 3 * d, d)) return cuda_fail("qkv upload failed");
    lw.bqkv = up_f32(bqkv);
    if (!gemm_w(lw.o, next(), d, d)) return cuda_fail("o upload failed");
    lw.bo = up_f32(next());
    lw.ln2g = up_f32(next());
    lw.ln2b = up_f32(next());
    if (!gemm_w(lw.fc1, next(), g->d_ffn, d)) return cuda_fail("fc1 upload failed");
    lw.b1 = up_f32(next());
    if (!gemm_w(lw.fc2, next(), d, g->d_ffn)) return cuda_fail("fc2 upload failed");
    lw.b2 = up_f32(next());
  }
  e->lnpg = up_f32(next());
  e->lnpb = up_f32(next());
  e->ln_fuse = L > 0 && e->kind != KIND_TF32 && gemm_ln_supported(e->layers[0].o, e->num_sms) &&
               gemm_ln_supported(e->layers[0].fc2, e->num_sms);
  if (g->proj1_out) {
    if (!gemm_w(e->p1, next(), g->proj1_out, d)) return cuda_fail("proj1 upload failed");
    e->bp1 = up_f32(next());
    if (!gemm_w(e->p2, next(), g->proj2_out, g->proj1_out)) return cuda_fail("proj2 upload failed");
    e->bp2 = up_f32(next());
  }
  if (g->adapter_hidden) {
    const int H = g->adapter_hidden, K = g->proj2_out;
    auto wg = next();
    auto wu = next();
    std::vector<float> r((size_t)2 * H * K);
    for (int j = 0; j < H / 16; ++j)
      for (int i = 0; i < 16; ++i) {
        memcpy(&r[((size_t)32 * j + i) * K], &wg[((size_t)16 * j + i) * K], K * 4);
        memcpy(&r[((size_t)32 * j + 16 + i) * K], &wu[((size_t)16 * j + i) * K], K * 4);
      }
    if (!gemm_w(e->gu, r, 2 * H, K)) return cuda_fail("adapter gate/up upload failed");
    if (!gemm_w(e->down, next(), g->adapter_out, H)) return cuda_fail("adapter down upload failed");
  }
  e->pe_rows = pe_rows;
  e->pe = up_f32(build_pe(pe_rows, d));
  e->mel_tab = static_cast<MelTables*>(slab_take(e, sizeof(MelTables)));
  if (!e->mel_tab) return bad(fail(e, ASR_E_NOMEM, "slab exhausted"));
  note(launch_mel_tables(g->n_mels, e->mel_tab, st), "mel table kernel launch");
  e->status = static_cast<int*>(slab_take(e, 256));
  if (!e->status) return bad(fail(e, ASR_E_NOMEM, "slab exhausted"));
  note(cudaMemsetAsync(e->status, 0, 256, st), "cudaMemsetAsync (status word)");
  note(cudaStreamSynchronize(st), "cudaStreamSynchronize");
  if (cerr != cudaSuccess) return cuda_fail("weight repack");
  if (!e->pe || !e->c2.ptr || !e->c2b || !e->c3b || !e->lnpg || !e->lnpb) return bad(fail(e, ASR_E_NOMEM, "slab exhausted"));
  *out = e;
  return ASR_OK;
}

}  // extern "C"

namespace {

size_t sk_flags_bytes(const asr_enc* e) { return ((size_t)e->num_sms * 8 * 4 + 255) / 256 * 256; }
// LayerNorm epilogue: one arrival counter per 32 rows, and per row two
// partial statistics (16 bytes each) per 256-column n-tile.
size_t ln_count_bytes(int64_t T) { return ((size_t)(T + 31) / 32 * 4 + 255) / 256 * 256; }
int ln_parts(const asr_enc* e) { return 2 * ((e->g.d_model + 255) / 256); }

bool make_plan(const asr_enc* e, int64_t n, int B, Plan* p) {
  const size_t es = e->es;  // activation element size
  const asr_geometry* g = &e->g;
  const int64_t tc = tokens_per_clip(g, n);
  if (tc <= 0 || B <= 0) return false;
  p->n = n;
  p->B = B;
  p->Tc = tc;
  p->T = tc * B;
  p->F = (int)(n / g->hop);
  const int64_t w = g->window_tokens ? g->window_tokens : tc;
  p->nwin_clip = (int)((tc + w - 1) / w);
  p->nwin = p->nwin_clip * B;
  p->max_win = (int)std::min<int64_t>(w, tc);
  const int d = g->d_model;
  p->Tpad = p->T;
  p->n_total = n * B;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    off = align_up(off, 1024);
    size_t r = off;
    off += bytes;
    return r;
  };
  p->off_clipmax = take((size_t)B * 4);
  p->off_cu = take((size_t)(p->nwin + 1) * 4);
  p->off_mel = take((size_t)B * g->n_mels * p->F * 4);
  if (g->stem == ASR_STEM_CONV2D_CHUNKED) {
    p->chunks = (int)(B * (p->F / g->chunk_frames));
    p->T1 = (int)conv_len(g->chunk_frames, 3, 2, 1); p->F1 = (int)conv_len(g->n_mels, 3, 2, 1);
    p->T2 = (int)conv_len(p->T1, 3, 2, 1); p->F2 = (int)conv_len(p->F1, 3, 2, 1);
    p->T3 = (int)conv_len(p->T2, 3, 2, 1); p->F3 = (int)conv_len(p->F2, 3, 2, 1);
    const size_t C = g->conv_ch;
    set_stem_rows(e->packed, p);
    p->off_a1 = take((size_t)p->rows1 * 16 * es);
    p->off_c1 = take((size_t)p->rows1 * C * es);
    p->off_c2 = take((size_t)p->rows2 * C * es);
    p->off_c3 = take((size_t)p->T * p->F3 * C * es);
  } else {
    p->off_melT = take((size_t)B * p->F * g->n_mels * es);
    p->off_c1 = take((size_t)B * p->F * d * es);
  }
  p->off_x = take((size_t)p->T * d * 4);
  p->off_h = take((size_t)p->T * d * es);
  p->off_qkv = take((size_t)p->T * 3 * d * es);
  p->off_att = take((size_t)p->T * d * es);
  p->off_ff = take((size_t)p->T * g->d_ffn * es);
  if (g->proj1_out) {
    p->off_p1 = take((size_t)p->T * g->proj1_out * es);
    p->off_p2 = take((size_t)p->T * g->proj2_out * es);
  }
  if (g->adapter_hidden) p->off_gu = take((size_t)p->T * g->adapter_hidden * es);
  p->tap_bytes[ASR_TAP_MEL] = (size_t)B * g->n_mels * p->F * 4;
  p->tap_bytes[ASR_TAP_STEM] = p->tap_bytes[ASR_TAP_LAYER0] = p->tap_bytes[ASR_TAP_ENCODER] = (size_t)p->T * d * 4;
  p->tap_bytes[ASR_TAP_HEAD] = g->proj2_out ? (size_t)p->T * g->proj2_out * 4 : 0;
  for (int t = 0; t < ASR_TAP_COUNT; ++t)
    if ((e->taps >> t) & 1u) p->off_tap[t] = take(p->tap_bytes[t]);
  p->off_pcm = take((size_t)B * n * 4);
  p->off_out = take((size_t)p->T * d_out(g) * 4);
  p->off_skflags = take(sk_flags_bytes(e));
  if (e->ln_fuse) {
    p->off_lncnt = take(ln_count_bytes(p->T));
    p->off_lnpart = take((size_t)p->T * ln_parts(e) * 16);
  }
  p->total = align_up(off, 1024);
  return true;
}

// Plan of a variable-length batch of the conv2d stem: clip b has ns[b]
// samples.  Conv buffers hold every chunk at full size (a short last chunk
// padded); conv_out writes padded token rows, compacted into the clips'
// packed rows before the tower.
//  s_offs, lefts (optional): clip b's samples start at pcm + s_offs[b] with
//  lefts[b] real samples before them (streamed windows); by default the clips
//  are packed back to back with no history.
bool make_plan_varlen(const asr_enc* e, const int64_t* ns, int B, Plan* p, const int64_t* s_offs = nullptr,
                      const int* lefts = nullptr) {
  const size_t es = e->es;  // activation element size
  const asr_geometry* g = &e->g;
  if (g->stem != ASR_STEM_CONV2D_CHUNKED || !ns || B <= 0) return false;
  p->varlen = true;
  p->B = B;
  p->n = -1;
  p->F = 0;
  p->Tc = 0;
  const int cf = g->chunk_frames;
  const int t3 = (int)chunk_tokens(cf);
  const int w = g->window_tokens;
  p->T1 = (int)conv_len(cf, 3, 2, 1); p->F1 = (int)conv_len(g->n_mels, 3, 2, 1);
  p->T2 = (int)conv_len(p->T1, 3, 2, 1); p->F2 = (int)conv_len(p->F1, 3, 2, 1);
  p->T3 = (int)conv_len(p->T2, 3, 2, 1); p->F3 = (int)conv_len(p->F2, 3, 2, 1);
  p->clips.assign(B, VarClip{});
  int64_t s = 0, f = 0, groups = 0, ch = 0, tok = 0, win = 0;
  int maxseg = 0;
  p->has_short = false;
  for (int b = 0; b < B; ++b) {
    const int64_t n = ns[b];
    // a clip with real history before it (a streamed window) needs only one hop
    const int64_t tb = (lefts && lefts[b] >= g->n_fft / 2) ? tokens_from_frames(g, n / g->hop) : tokens_per_clip(g, n);
    if (tb <= 0) return false;
    const int64_t F = n / g->hop, K = (F + cf - 1) / cf;
    const int64_t W = w ? (tb + w - 1) / w : 1;
    if (F % cf) p->has_short = true;
    VarClip& v = p->clips[b];
    v.s_off = s_offs ? s_offs[b] : s; v.n = n; v.f_off = f; v.frames = (int)F; v.g_off = (int)groups;
    v.left = lefts ? lefts[b] : 0;
    v.chunk_off = (int)ch; v.chunks = (int)K; v.tok_off = (int)tok; v.tokens = (int)tb;
    v.win_off = (int)win; v.wins = (int)W;
    maxseg = std::max<int>(maxseg, (int)(w ? std::min<int64_t>(w, tb) : tb));
    s += n; f += F; groups += mel_groups(F); ch += K; tok += tb; win += W;
    if (s > (1LL << 40) || ch * t3 > 0x7FFFFFFFLL / 8 || groups > 0x7FFFFFFF || win > 0x7FFFFFF) return false;
  }
  p->n_total = s;
  p->Ftot = f;
  p->n_groups = (int)groups;
  p->chunks = (int)ch;
  p->Tpad = ch * t3;
  p->T = tok;
  p->nwin = (int)win;
  p->max_win = maxseg;
  p->nwin_clip = 0;
  const int d = g->d_model;
  const size_t C = g->conv_ch;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    off = align_up(off, 1024);
    size_t r = off;
    off += bytes;
    return r;
  };
  p->off_clipmax = take((size_t)B * 4);
  p->off_mclips = take((size_t)B * sizeof(MelClip));
  p->off_chunkd = take((size_t)p->chunks * sizeof(ChunkDesc));
  p->off_cu = take((size_t)(p->nwin + 1) * 4);
  p->off_mel = take((size_t)g->n_mels * p->Ftot * 4);
  set_stem_rows(e->packed, p);
  p->off_a1 = take((size_t)p->rows1 * 16 * es);
  p->off_c1 = take((size_t)p->rows1 * C * es);
  p->off_c2 = take((size_t)p->rows2 * C * es);
  p->off_c3 = take((size_t)p->Tpad * p->F3 * C * es);
  p->off_xpad = take((size_t)p->Tpad * d * 4);
  p->off_x = take((size_t)p->T * d * 4);
  p->off_h = take((size_t)p->T * d * es);
  p->off_qkv = take((size_t)p->T * 3 * d * es);
  p->off_att = take((size_t)p->T * d * es);
  p->off_ff = take((size_t)p->T * g->d_ffn * es);
  if (g->proj1_out) {
    p->off_p1 = take((size_t)p->T * g->proj1_out * es);
    p->off_p2 = take((size_t)p->T * g->proj2_out * es);
  }
  if (g->adapter_hidden) p->off_gu = take((size_t)p->T * g->adapter_hidden * es);
  p->tap_bytes[ASR_TAP_MEL] = 0;  // the mel tap covers uniform batches only
  p->tap_bytes[ASR_TAP_STEM] = p->tap_bytes[ASR_TAP_LAYER0] = p->tap_bytes[ASR_TAP_ENCODER] = (size_t)p->T * d * 4;
  p->tap_bytes[ASR_TAP_HEAD] = g->proj2_out ? (size_t)p->T * g->proj2_out * 4 : 0;
  for (int t = 0; t < ASR_TAP_COUNT; ++t)
    if (((e->taps >> t) & 1u) && p->tap_bytes[t]) p->off_tap[t] = take(p->tap_bytes[t]);
  p->off_pcm = take((size_t)p->n_total * 4);
  p->off_out = take((size_t)p->T * d_out(g) * 4);
  p->off_skflags = take(sk_flags_bytes(e));
  if (e->ln_fuse) {
    p->off_lncnt = take(ln_count_bytes(p->T));
    p->off_lnpart = take((size_t)p->T * ln_parts(e) * 16);
  }
  p->total = align_up(off, 1024);
  return true;
}

// The plan of a batch: per-clip sizes `ns` (variable length), or B clips of
// n samples (uniform when n is whole chunks, else the variable-length plan
// with every clip of n samples).
bool plan_for(const asr_enc* e, const int64_t* ns, int64_t n, int B, Plan* p) {
  if (ns) return make_plan_varlen(e, ns, B, p);
  if (B <= 0) return false;
  if (uniform_ok(&e->g, n)) return make_plan(e, n, B, p);
  if (e->g.stem != ASR_STEM_CONV2D_CHUNKED) return false;
  std::vector<int64_t> v(B, n);
  return make_plan_varlen(e, v.data(), B, p);
}

asr_status gemm(asr_enc* e, const CUtensorMap* amap, const ConvGather* cg, const GemmB& w, long long M, void* out,
                long long ldo, const float* bias, const float* pe, int period, int epi, cudaStream_t st,
                const CUtensorMap* omap, const ConvBox* box = nullptr, int zero_period = 0, int zero_from = 0,
                int* sk_flags = nullptr, const float* ln_g = nullptr, const float* ln_b = nullptr,
                const Plan* plan = nullptr, char* ws = nullptr, int ln_epoch = 0, int force_bn = 0) {
  // ln_g / ln_b: residual update followed by the LayerNorm (gamma, beta) of
  // the updated rows into h (EPI_LN; the plan and workspace give its buffers,
  // ln_epoch counts the earlier such launches of the forward)
  // fp32 operands: every output of the engine is fp32
  if (e->kind == KIND_TF32 && !(epi & (EPI_OUT_F32 | EPI_RESID))) epi |= EPI_OUT_F32;
  GemmParams p;
  memset(&p, 0, sizeof p);
  p.M = (int)M;
  p.out = out;
  p.ldo = ldo;
  p.bias = bias;
  p.pe = pe;
  p.pe_period = period;
  if (cg) p.g = *cg;
  p.status = e->status;
  p.limit_ns = kWaitLimitNs;
  p.zero_period = zero_period;
  p.zero_from = zero_from;
  p.sk_flags = sk_flags;  // stream-K allowed (residual epilogue, the launcher decides)
  if (ln_g) {
    epi |= EPI_LN;
    p.sk_flags = nullptr;
    p.ln_gamma = ln_g;
    p.ln_beta = ln_b;
    p.ln_eps = e->g.ln_eps;
    p.ln_count = reinterpret_cast<int*>(ws + plan->off_lncnt);
    p.ln_part = reinterpret_cast<float*>(ws + plan->off_lnpart);
    p.ln_h = ws + plan->off_h;
    p.ln_epoch = ln_epoch;
  }
  int bn;
  const CUtensorMap* amap3 = box ? nullptr : e->maps.companion3(amap);
  if (box) {
    p.conv_box = 1;
    p.cb = *box;
    bn = e->kind == KIND_TF32 ? gemm_pick_bn_tf32(box->n_sub * 128, w.N, e->num_sms)
                              : gemm_pick_bn_conv(box->n_sub, w.N, e->num_sms);
  } else {
    bn = e->kind == KIND_TF32 ? gemm_pick_bn_tf32((int)M, w.N, e->num_sms)
                              : gemm_pick_bn((int)M, w.N, e->num_sms, cg != nullptr);
  }
  if (force_bn) bn = force_bn;
  cudaError_t r = launch_gemm(amap, w, p, epi, bn, e->num_sms, st, omap, amap3);
  if (r != cudaSuccess) return fail(e, ASR_E_CUDA, "gemm launch (N=%d K=%d M=%lld epi=%d bn=%d): %s", w.N, w.K, M, epi, bn, cudaGetErrorString(r));
  return ASR_OK;
}

#define ASR_TRY(x)                 \
  do {                             \
    asr_status _s = (x);           \
    if (_s != ASR_OK) return _s;   \
  } while (0)
#define ASR_LAUNCH(e, x)                                                                                     \
  do {                                                                                                       \
    cudaError_t _r = (x);                                                                                    \
    if (_r != cudaSuccess) return fail((e), ASR_E_CUDA, "%s: %s", #x, cudaGetErrorString(_r));               \
  } while (0)

enum ProfClass { PC_MEL, PC_CONV1, PC_GEMM_CONV, PC_GEMM_CONVOUT, PC_GEMM_QKV, PC_GEMM_O, PC_GEMM_FC1, PC_GEMM_FC2,
                 PC_GEMM_HEAD, PC_GEMM_ADAPTER, PC_LN, PC_ATTN, PC_MISC, PC_COUNT };
const char* const kProfNames[PC_COUNT] = {"log_mel", "conv1", "gemm_conv", "gemm_conv_out", "gemm_qkv", "gemm_o",
                                          "gemm_fc1", "gemm_fc2", "gemm_head", "gemm_adapter", "layer_norm",
                                          "attention", "misc"};

void prof_begin(asr_enc* e, int cls, cudaStream_t st) {
  ++e->launches;
  if (!e->prof) return;
  while (e->ev_used + 2 > e->ev_pool.size()) {
    cudaEvent_t ev;
    if (cudaEventCreate(&ev) != cudaSuccess) return;
    e->ev_pool.push_back(ev);
  }
  e->prof_recs.push_back({cls, e->ev_used});
  cudaEventRecord(e->ev_pool[e->ev_used], st);
  e->ev_used += 2;
}
void prof_end(asr_enc* e, cudaStream_t st) {
  if (!e->prof || e->prof_recs.empty()) return;
  cudaEventRecord(e->ev_pool[e->prof_recs.back().second + 1], st);
}
#define ASR_K(cls, stmt)          \
  do {                            \
    prof_begin(e, (cls), st);     \
    stmt;                         \
    prof_end(e, st);              \
  } while (0)

asr_status ensure_maps(asr_enc* e, const Plan& p, char* ws) {
  ActMaps& m = e->maps;
  if (m.ws == ws && m.n == p.n && m.batch == p.B && m.T == p.T && m.chunks == p.chunks && m.taps == e->taps) return ASR_OK;
  const asr_geometry* g = &e->g;
  const int d = g->d_model, k = e->kind;
  const bool f32 = k == KIND_TF32;  // fp32 activations between the GEMMs
  // (the qkv map feeds the tcgen05 attention, which takes bf16 operands)
  bool ok = (f32 || make_tmap_qkv(&m.qkv, ws + p.off_qkv, p.T, g->n_heads)) &&
            make_tmap_act(k, &m.h, ws + p.off_h, p.T, d, d, 128) &&
            make_tmap_act(k, &m.att, ws + p.off_att, p.T, d, d, 128) &&
            make_tmap_act(k, &m.ff, ws + p.off_ff, p.T, g->d_ffn, g->d_ffn, 128);
  if (ok && g->stem == ASR_STEM_CONV2D_CHUNKED) {
    const int C = g->conv_ch;
    ok = make_tmap_act(k, &m.c3, ws + p.off_c3, p.Tpad, (size_t)p.F3 * C, (size_t)p.F3 * C, 128) &&
         make_tmap_act(k, &m.a1, ws + p.off_a1, (size_t)p.rows1, 16, 16, 128);
    // packed: one image of chunks x S2 rows (planes: [4][chunks * S2][F1 / 2][C])
    if (ok && e->box2)
      ok = e->packed   ? make_tmap_convphase(&m.cin2, ws + p.off_c1, C, p.F1 / 2, p.chunks * p.S2, 4, p.F2, 128 / p.F2, k)
           : e->phase2 ? make_tmap_convphase(&m.cin2, ws + p.off_c1, C, p.F1 / 2, p.T1 / 2, 4 * p.chunks, p.F2, 128 / p.F2, k)
                       : make_tmap_convbox(&m.cin2, ws + p.off_c1, C, p.F1, p.T1, p.chunks, p.F2, 2, 128 / p.F2, 2, k);
    if (ok && e->box3)
      ok = e->packed ? make_tmap_convbox(&m.cin3, ws + p.off_c2, C, p.F2, p.chunks * p.S2, 1, p.F3, 2, 128 / p.F3, 2, k)
                     : make_tmap_convbox(&m.cin3, ws + p.off_c2, C, p.F2, p.T2, p.chunks, p.F3, 2, 128 / p.F3, 2, k);
  } else if (ok) {
    ok = make_tmap_convbox(&m.cin2, ws + p.off_melT, g->n_mels, 1, p.F, p.B, 1, 1, 128, 1, k) &&
         make_tmap_convbox(&m.cin3, ws + p.off_c1, d, 1, p.F, p.B, 1, 1, 128, 2, k);
  }
  if (ok && g->proj1_out)
    ok = make_tmap_act(k, &m.p1, ws + p.off_p1, p.T, g->proj1_out, g->proj1_out, 128) &&
         make_tmap_act(k, &m.p2, ws + p.off_p2, p.T, g->proj2_out, g->proj2_out, 128) &&
         make_tmap_out(&m.o_p1, ws + p.off_p1, p.T, g->proj1_out, g->proj1_out, f32) &&
         make_tmap_out(&m.o_p2, ws + p.off_p2, p.T, g->proj2_out, g->proj2_out, f32);
  if (ok)
    ok = make_tmap_out(&m.o_x, ws + p.off_x, p.T, d, d, true) &&
         make_tmap_out(&m.o_qkv, ws + p.off_qkv, p.T, 3 * d, 3 * d, f32) &&
         make_tmap_out(&m.o_ff, ws + p.off_ff, p.T, g->d_ffn, g->d_ffn, f32);
  if (ok && g->stem == ASR_STEM_CONV2D_CHUNKED)
    ok = make_tmap_out(&m.o_c1, ws + p.off_c1, (unsigned long long)p.rows1, g->conv_ch, g->conv_ch, f32) &&
         make_tmap_out(&m.o_c2, ws + p.off_c2, (unsigned long long)p.rows2, g->conv_ch, g->conv_ch, f32) &&
         make_tmap_out(&m.o_c3, ws + p.off_c3, (unsigned long long)p.chunks * p.T3 * p.F3, g->conv_ch, g->conv_ch, f32);
  else if (ok)
    ok = make_tmap_out(&m.o_c1, ws + p.off_c1, (unsigned long long)p.B * p.F, d, d, f32);
  if (ok && g->adapter_hidden) ok = make_tmap_act(k, &m.gu, ws + p.off_gu, p.T, g->adapter_hidden, g->adapter_hidden, 128);
  // QKV split: the CTA-pair launch takes whole 256-row blocks; with T % 256
  // rows left over (the 16 x 30 s batch: 6240 = 24 x 256 + 96) it would run
  // one more wave of tiles a third full, which the one-SM tail launch replaces
  m.qkv_main = 0;
  if (ok && !f32 && p.T > 256 && p.T % 256 && d % 128 == 0) {
    const int64_t mm = p.T / 256 * 256;
    ok = make_tmap_act(k, &m.h_tail, ws + p.off_h + (size_t)mm * d * e->es, p.T - mm, d, d, 128) &&
         make_tmap_out(&m.o_qkv_tail, ws + p.off_qkv + (size_t)mm * 3 * d * e->es, p.T - mm, 3 * d, 3 * d, false);
    if (ok) m.qkv_main = mm;
  }
  m.n3 = 0;
  if (ok)
    ok = m.add3(&m.h, ws + p.off_h, p.T, d, k) && m.add3(&m.att, ws + p.off_att, p.T, d, k) &&
         m.add3(&m.ff, ws + p.off_ff, p.T, g->d_ffn, k);
  if (ok && g->stem == ASR_STEM_CONV2D_CHUNKED)
    ok = m.add3(&m.c3, ws + p.off_c3, p.Tpad, (unsigned long long)p.F3 * g->conv_ch, k);
  if (ok && g->proj1_out)
    ok = m.add3(&m.p1, ws + p.off_p1, p.T, g->proj1_out, k) && m.add3(&m.p2, ws + p.off_p2, p.T, g->proj2_out, k);
  if (ok && g->adapter_hidden) ok = m.add3(&m.gu, ws + p.off_gu, p.T, g->adapter_hidden, k);
  if (!ok) {
    m.ws = nullptr;
    return fail(e, ASR_E_CUDA, "TMA descriptor encoding failed (workspace alignment?)");
  }
  m.ws = ws;
  m.n = p.n;
  m.T = p.T;
  m.chunks = p.chunks;
  m.batch = p.B;
  m.taps = e->taps;
  return ASR_OK;
}

asr_status run_forward(asr_enc* e, const float* pcm, const Plan& p, float* out, char* ws, cudaStream_t st) {
  const asr_geometry* g = &e->g;
  const int d = g->d_model;
  ASR_TRY(ensure_maps(e, p, ws));
  unsigned* clip_max = reinterpret_cast<unsigned*>(ws + p.off_clipmax);
  int* cu = reinterpret_cast<int*>(ws + p.off_cu);
  float* mel = reinterpret_cast<float*>(ws + p.off_mel);
  float* x = reinterpret_cast<float*>(ws + p.off_x);
  // activations between the GEMMs: bf16, or fp32 on the tf32 path
  const bool f32 = e->kind == KIND_TF32, f16 = e->kind == KIND_F16;
  const int RE = kind_row_elems(e->kind), KST = RE / 4;  // conv channel block, MMA step (elements)
  void* h = ws + p.off_h;
  void* qkv = ws + p.off_qkv;
  void* att = ws + p.off_att;
  void* ff = ws + p.off_ff;
  auto tap = [&](int t) -> float* { return ((e->taps >> t) & 1u) ? reinterpret_cast<float*>(ws + p.off_tap[t]) : nullptr; };

  e->launches = 0;
  e->ev_used = 0;
  e->prof_recs.clear();
  ASR_LAUNCH(e, cudaMemsetAsync(e->status, 0, 4, st));
  ASR_LAUNCH(e, cudaMemsetAsync(clip_max, 0, (size_t)p.B * 4, st));
  if (e->maps.qkv_main && !e->aux_st) {
    if (cudaStreamCreateWithFlags(&e->aux_st, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&e->ev_fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&e->ev_join, cudaEventDisableTiming) != cudaSuccess)
      return fail(e, ASR_E_CUDA, "side stream / events for the split QKV projection");
  }
  int* skf = reinterpret_cast<int*>(ws + p.off_skflags);
  ASR_LAUNCH(e, cudaMemsetAsync(skf, 0, sk_flags_bytes(e), st));
  // LayerNorm epilogue of fc2 (16-bit tower): the next block's LN1, or the
  // head's LayerNorm
  const bool lnf = e->ln_fuse && e->ln_fuse_on && !f32;
  if (lnf) ASR_LAUNCH(e, cudaMemsetAsync(ws + p.off_lncnt, 0, ln_count_bytes(p.T), st));
  MelClip* mclips = reinterpret_cast<MelClip*>(ws + p.off_mclips);
  ChunkDesc* chunkd = reinterpret_cast<ChunkDesc*>(ws + p.off_chunkd);
  if (!p.varlen) {
    const int w = g->window_tokens ? g->window_tokens : (int)p.Tc;
    ASR_K(PC_MISC, ASR_LAUNCH(e, launch_fill_windows(cu, p.B, (int)p.Tc, w, p.nwin_clip, st)));
    ASR_K(PC_MEL, ASR_LAUNCH(e, launch_log_mel(pcm, p.n, p.B, g->n_mels, e->mel_tab, mel, clip_max, st)));
    if (float* t = tap(ASR_TAP_MEL)) ASR_K(PC_MISC, ASR_LAUNCH(e, launch_mel_normalize(mel, clip_max, (long long)g->n_mels * p.F, p.B, t, st)));
  } else {
    // per-clip descriptors, chunk descriptors and window offsets, 32 clips a launch
    const int t3 = p.T3;
    for (int b0 = 0; b0 < p.B; b0 += kVarClipsPerLaunch) {
      VarClipBatch vb;
      vb.first = b0;
      vb.count = std::min(kVarClipsPerLaunch, p.B - b0);
      for (int i = 0; i < vb.count; ++i) vb.c[i] = p.clips[b0 + i];
      const int last = b0 + vb.count == p.B ? 1 : 0;
      ASR_K(PC_MISC, ASR_LAUNCH(e, launch_varlen_fill(vb, g->chunk_frames, g->window_tokens, t3, mclips, chunkd, cu, last,
                                                      p.nwin, (int)p.T, st)));
    }
    MelArgs ma = {};
    ma.pcm = pcm;
    ma.mel = mel;
    ma.clip_max = clip_max;
    ma.n_mels = g->n_mels;
    ma.batch = p.B;
    ma.n_groups = p.n_groups;
    ma.clips = mclips;
    ASR_K(PC_MEL, ASR_LAUNCH(e, launch_log_mel(ma, e->mel_tab, st)));
  }

  if (g->stem == ASR_STEM_CONV2D_CHUNKED) {
    const int C = g->conv_ch;
    void* c1 = ws + p.off_c1;
    void* c2 = ws + p.off_c2;
    void* c3 = ws + p.off_c3;
    void* a1 = ws + p.off_a1;
    // row layout of conv1's output: 0 plain, 1 parity planes per chunk, 2 packed
    const int lay1 = e->packed ? 2 : (e->phase2 ? 1 : 0);
    if (!p.varlen)
      ASR_K(PC_CONV1, ASR_LAUNCH(e, launch_conv1_im2col(mel, clip_max, p.B, g->n_mels, p.F, g->chunk_frames, lay1, a1,
                                                        e->kind, st)));
    else
      ASR_K(PC_CONV1, ASR_LAUNCH(e, launch_conv1_im2col_varlen(mel, clip_max, p.chunks, g->n_mels, g->chunk_frames, lay1,
                                                               chunkd, mclips, a1, e->kind, st)));
    // packed: the zero row j = S2 - 1 of every chunk in every plane stays zero
    const int fh = p.F1 / 2;
    ASR_K(PC_CONV1, ASR_TRY(gemm(e, &e->maps.a1, nullptr, e->c1, p.rows1, c1, C, e->c1b, nullptr, 1, EPI_GELU, st,
                                 &e->maps.o_c1, nullptr, e->packed ? p.S2 * fh : 0, e->packed ? (p.S2 - 1) * fh : 0)));
    if (p.has_short)
      ASR_K(PC_MISC, ASR_LAUNCH(e, launch_mask_short_chunks(c1, chunkd, p.chunks, g->chunk_frames, 1, p.T1, p.F1, C, lay1,
                                                            p.S2, e->es, st)));
    const int CB = (C + RE - 1) / RE;
    const int k_last = (C - RE * (CB - 1) + KST - 1) / KST;
    if (e->box2) {
      // packed: one image of chunks x S2 output rows, the last row of every
      // chunk written as zeros (conv3's padding)
      const int TR = 128 / p.F2, To = e->packed ? p.chunks * p.S2 : p.T2, tpi = (To + TR - 1) / TR;
      ConvBox b2 = {TR, p.F2, To, tpi, e->packed ? tpi : p.chunks * tpi, 2, 2, 1, 1, 3, CB, e->phase2 ? 1 : 0, k_last};
      ASR_K(PC_GEMM_CONV, ASR_TRY(gemm(e, &e->maps.cin2, nullptr, e->c2, p.rows2, c2, C, e->c2b, nullptr, 1, EPI_GELU, st,
                                       &e->maps.o_c2, &b2, e->packed ? p.S2 * p.F2 : 0, e->packed ? p.T2 * p.F2 : 0)));
    } else {
      ConvGather cg2 = {static_cast<const bf16*>(c1), p.T1, p.F1, C, p.T2, p.F2, 2, 2, 3, 3, 1, 1};
      ASR_K(PC_GEMM_CONV, ASR_TRY(gemm(e, nullptr, &cg2, e->c2, (long long)p.chunks * p.T2 * p.F2, c2, C, e->c2b, nullptr, 1, EPI_GELU, st, &e->maps.o_c2)));
    }
    if (p.has_short)
      ASR_K(PC_MISC, ASR_LAUNCH(e, launch_mask_short_chunks(c2, chunkd, p.chunks, g->chunk_frames, 2, p.T2, p.F2, C,
                                                            e->packed ? 2 : 0, p.S2, e->es, st)));
    if (e->box3) {
      // packed: conv3 output row o = 13 c + t reads conv2 rows 26 c + 2 t - 1 ..
      // + 1 of the one image, whose zero rows are the chunks' padding
      const int TR = 128 / p.F3, To = e->packed ? p.chunks * p.T3 : p.T3, tpi = (To + TR - 1) / TR;
      ConvBox b3 = {TR, p.F3, To, tpi, e->packed ? tpi : p.chunks * tpi, 2, 2, 1, 1, 3, CB, 0, k_last};
      ASR_K(PC_GEMM_CONV, ASR_TRY(gemm(e, &e->maps.cin3, nullptr, e->c3, (long long)p.chunks * p.T3 * p.F3, c3, C, e->c3b, nullptr, 1, EPI_GELU, st, &e->maps.o_c3, &b3)));
    } else {
      ConvGather cg3 = {static_cast<const bf16*>(c2), p.T2, p.F2, C, p.T3, p.F3, 2, 2, 3, 3, 1, 1};
      ASR_K(PC_GEMM_CONV, ASR_TRY(gemm(e, nullptr, &cg3, e->c3, (long long)p.chunks * p.T3 * p.F3, c3, C, e->c3b, nullptr, 1, EPI_GELU, st, &e->maps.o_c3)));
    }
    if (!p.varlen) {
      ASR_K(PC_GEMM_CONVOUT, ASR_TRY(gemm(e, &e->maps.c3, nullptr, e->cout, p.T, x, d, nullptr, e->pe, p.T3, EPI_OUT_F32 | EPI_PE, st, nullptr)));
    } else {
      float* xpad = reinterpret_cast<float*>(ws + p.off_xpad);
      ASR_K(PC_GEMM_CONVOUT, ASR_TRY(gemm(e, &e->maps.c3, nullptr, e->cout, p.Tpad, xpad, d, nullptr, e->pe, p.T3, EPI_OUT_F32 | EPI_PE, st, nullptr)));
      ASR_K(PC_MISC, ASR_LAUNCH(e, launch_compact_tokens(xpad, x, chunkd, p.chunks, p.T3, d, st)));
    }
  } else {
    if (p.Tc > e->pe_rows) return fail(e, ASR_E_UNSUPPORTED, "conv1d stem: %lld positions > %d", (long long)p.Tc, e->pe_rows);
    void* melT = ws + p.off_melT;
    void* c1 = ws + p.off_c1;
    ASR_K(PC_MISC, ASR_LAUNCH(e, launch_mel_normalize_transpose(mel, clip_max, p.B, g->n_mels, p.F, melT, e->kind, st)));
    const int tpi1 = (p.F + 127) / 128, tpi2 = (int)((p.Tc + 127) / 128);
    const int CB1 = (g->n_mels + RE - 1) / RE, CBd = (d + RE - 1) / RE;
    ConvBox b1 = {128, 1, p.F, tpi1, p.B * tpi1, 1, 1, 1, 0, 1, CB1, 0, (g->n_mels - RE * (CB1 - 1) + KST - 1) / KST};
    ASR_K(PC_GEMM_CONV, ASR_TRY(gemm(e, &e->maps.cin2, nullptr, e->c2, (long long)p.B * p.F, c1, d, e->c2b, nullptr, 1, EPI_GELU, st, &e->maps.o_c1, &b1)));
    ConvBox b2 = {128, 1, (int)p.Tc, tpi2, p.B * tpi2, 2, 1, 1, 0, 1, CBd, 0, (d - RE * (CBd - 1) + KST - 1) / KST};
    ASR_K(PC_GEMM_CONV, ASR_TRY(gemm(e, &e->maps.cin3, nullptr, e->c3, p.T, x, d, e->c3b, e->pe, (int)p.Tc, EPI_GELU | EPI_OUT_F32 | EPI_PE, st, nullptr, &b2)));
  }
  if (float* t = tap(ASR_TAP_STEM)) ASR_LAUNCH(e, cudaMemcpyAsync(t, x, (size_t)p.T * d * 4, cudaMemcpyDeviceToDevice, st));

  for (int l = 0; l < g->n_layers; ++l) {
    const LayerW& lw = e->layers[l];
    if (l == 0 || !lnf) ASR_K(PC_LN, ASR_LAUNCH(e, launch_layer_norm(x, lw.ln1g, lw.ln1b, p.T, d, g->ln_eps, h, e->kind, st)));
    if (e->maps.qkv_main) {
      // rows [0, main) on CTA-pair tiles; the last T % 256 rows on one-SM
      // tiles on the side stream, whose CTAs take the SMs that the pair
      // launch leaves idle in its last wave; joined before the attention
      const int64_t mm = e->maps.qkv_main;
      void* qkv_tail = static_cast<char*>(qkv) + (size_t)mm * 3 * d * e->es;
      prof_begin(e, PC_GEMM_QKV, st);
      ASR_LAUNCH(e, cudaEventRecord(e->ev_fork, st));
      ASR_TRY(gemm(e, &e->maps.h, nullptr, lw.qkv, mm, qkv, 3 * d, lw.bqkv, nullptr, 1, 0, st, &e->maps.o_qkv));
      ASR_LAUNCH(e, cudaStreamWaitEvent(e->aux_st, e->ev_fork, 0));
      ++e->launches;
      ASR_TRY(gemm(e, &e->maps.h_tail, nullptr, lw.qkv, p.T - mm, qkv_tail, 3 * d, lw.bqkv, nullptr, 1, 0, e->aux_st,
                   &e->maps.o_qkv_tail, nullptr, 0, 0, nullptr, nullptr, nullptr, nullptr, nullptr, 0, 256));
      ASR_LAUNCH(e, cudaEventRecord(e->ev_join, e->aux_st));
      ASR_LAUNCH(e, cudaStreamWaitEvent(st, e->ev_join, 0));
      prof_end(e, st);
    } else {
      ASR_K(PC_GEMM_QKV, ASR_TRY(gemm(e, &e->maps.h, nullptr, lw.qkv, p.T, qkv, 3 * d, lw.bqkv, nullptr, 1, 0, st, &e->maps.o_qkv)));
    }
    if (f32)
      ASR_K(PC_ATTN, ASR_LAUNCH(e, launch_attention_f32(static_cast<const float*>(qkv), cu, p.nwin, p.max_win,
                                                        g->n_heads, static_cast<float*>(att), st)));
    else if (p.max_win <= 128)
      ASR_K(PC_ATTN, ASR_LAUNCH(e, launch_attention_tc(e->maps.qkv, qkv, cu, p.nwin, g->n_heads, att, e->status,
                                                       kWaitLimitNs, f16, st)));
    else
      ASR_K(PC_ATTN, ASR_LAUNCH(e, launch_attention_fa(e->maps.qkv, cu, p.nwin, p.max_win, g->n_heads, att, e->status,
                                                       kWaitLimitNs, f16, st)));
    // The out-projection keeps the separate LayerNorm: its K = d_model
    // mainloop is shorter than the LayerNorm epilogue, which would then
    // stall the tensor cores (measured slower than the two launches).
    ASR_K(PC_GEMM_O, ASR_TRY(gemm(e, &e->maps.att, nullptr, lw.o, p.T, x, d, lw.bo, nullptr, 1, EPI_RESID, st,
                                  &e->maps.o_x, nullptr, 0, 0, skf)));
    ASR_K(PC_LN, ASR_LAUNCH(e, launch_layer_norm(x, lw.ln2g, lw.ln2b, p.T, d, g->ln_eps, h, e->kind, st)));
    ASR_K(PC_GEMM_FC1, ASR_TRY(gemm(e, &e->maps.h, nullptr, lw.fc1, p.T, ff, g->d_ffn, lw.b1, nullptr, 1, EPI_GELU, st, &e->maps.o_ff)));
    // the LayerNorm that reads this update: the next layer's LN1, or the head's
    const bool last = l + 1 == g->n_layers;
    const float* nlg = !lnf ? nullptr : !last ? e->layers[l + 1].ln1g : g->proj1_out ? e->lnpg : nullptr;
    const float* nlb = !lnf ? nullptr : !last ? e->layers[l + 1].ln1b : e->lnpb;
    ASR_K(PC_GEMM_FC2, ASR_TRY(gemm(e, &e->maps.ff, nullptr, lw.fc2, p.T, x, d, lw.b2, nullptr, 1, EPI_RESID, st, &e->maps.o_x,
                                    nullptr, 0, 0, nlg ? nullptr : skf, nlg, nlb, &p, ws, l)));
    if (l == 0)
      if (float* t = tap(ASR_TAP_LAYER0)) ASR_LAUNCH(e, cudaMemcpyAsync(t, x, (size_t)p.T * d * 4, cudaMemcpyDeviceToDevice, st));
  }
  if (float* t = tap(ASR_TAP_ENCODER)) ASR_LAUNCH(e, cudaMemcpyAsync(t, x, (size_t)p.T * d * 4, cudaMemcpyDeviceToDevice, st));

  if (!g->proj1_out) {
    ASR_K(PC_LN, ASR_LAUNCH(e, launch_layer_norm(x, e->lnpg, e->lnpb, p.T, d, g->ln_eps, out, KIND_TF32, st)));
    return ASR_OK;
  }
  void* p1 = ws + p.off_p1;
  void* p2 = ws + p.off_p2;
  // Store map of the caller's output (plain stores if it is not 16-byte aligned).
  CUtensorMap o_out_map;
  const CUtensorMap* o_out = make_tmap_out(&o_out_map, out, p.T, d_out(g), d_out(g), true) ? &o_out_map : nullptr;
  if (!lnf) ASR_K(PC_LN, ASR_LAUNCH(e, launch_layer_norm(x, e->lnpg, e->lnpb, p.T, d, g->ln_eps, h, e->kind, st)));
  ASR_K(PC_GEMM_HEAD, ASR_TRY(gemm(e, &e->maps.h, nullptr, e->p1, p.T, p1, g->proj1_out, e->bp1, nullptr, 1, EPI_GELU, st, &e->maps.o_p1)));
  if (!g->adapter_hidden) {
    ASR_K(PC_GEMM_HEAD, ASR_TRY(gemm(e, &e->maps.p1, nullptr, e->p2, p.T, out, g->proj2_out, e->bp2, nullptr, 1, EPI_OUT_F32, st, o_out)));
    if (float* t = tap(ASR_TAP_HEAD)) ASR_LAUNCH(e, cudaMemcpyAsync(t, out, (size_t)p.T * g->proj2_out * 4, cudaMemcpyDeviceToDevice, st));
    return ASR_OK;
  }
  ASR_K(PC_GEMM_HEAD, ASR_TRY(gemm(e, &e->maps.p1, nullptr, e->p2, p.T, p2, g->proj2_out, e->bp2, nullptr, 1, 0, st, &e->maps.o_p2)));
  if (float* t = tap(ASR_TAP_HEAD)) {
    if (f32)
      ASR_LAUNCH(e, cudaMemcpyAsync(t, p2, (size_t)p.T * g->proj2_out * 4, cudaMemcpyDeviceToDevice, st));
    else
      ASR_K(PC_MISC, ASR_LAUNCH(e, launch_bf16_to_f32(p2, t, (long long)p.T * g->proj2_out, f16, st)));
  }
  void* gu = ws + p.off_gu;
  ASR_K(PC_GEMM_ADAPTER, ASR_TRY(gemm(e, &e->maps.p2, nullptr, e->gu, p.T, gu, g->adapter_hidden, nullptr, nullptr, 1, EPI_SWIGLU, st, nullptr)));
  ASR_K(PC_GEMM_ADAPTER, ASR_TRY(gemm(e, &e->maps.gu, nullptr, e->down, p.T, out, g->adapter_out, nullptr, nullptr, 1, EPI_OUT_F32, st, o_out)));
  return ASR_OK;
}

// Validates a forward of `B` clips, per-clip sizes `ns` (variable length) or
// n samples each, and builds its plan.
asr_status check_forward_args(asr_enc* e, const int64_t* ns, int64_t n, int B, const void* pcm, const void* out, void* ws,
                              size_t ws_bytes, Plan* p) {
  if (!e) return fail(nullptr, ASR_E_INVAL, "handle is NULL");
  if (!pcm || !out) return fail(e, ASR_E_INVAL, "pcm or out is NULL");
  if (B <= 0) return fail(e, ASR_E_INVAL, "batch must be > 0");
  const asr_geometry* g = &e->g;
  for (int b = 0; b < (ns ? B : 1); ++b) {
    const int64_t nb = ns ? ns[b] : n;
    if (nb <= g->n_fft / 2) return fail(e, ASR_E_INVAL, "clip %d: n_samples must exceed n_fft/2 (reflect padding)", b);
    if (g->stem == ASR_STEM_CONV1D && (nb % g->hop || (nb / g->hop) % 2))
      return fail(e, ASR_E_UNSUPPORTED, "conv1d stem: n_samples must be an even number of hops (%d samples)", g->hop);
  }
  if (ns && g->stem != ASR_STEM_CONV2D_CHUNKED)
    return fail(e, ASR_E_UNSUPPORTED, "variable-length batches need the chunked conv2d stem");
  if (!ns) {
    const int64_t T = tokens_per_clip(g, n) * B;
    if (T > 0x7FFFFFFFLL / 8 || (int64_t)B * n > (1LL << 40)) return fail(e, ASR_E_UNSUPPORTED, "batch too large");
  }
  if (!plan_for(e, ns, n, B, p)) return fail(e, ASR_E_UNSUPPORTED, "batch too large or sizes unsupported");
  if (p->varlen && ((e->taps >> ASR_TAP_MEL) & 1u))
    return fail(e, ASR_E_UNSUPPORTED, "the mel tap covers batches of whole chunks only");
  if (!ws || ws_bytes < p->total) return fail(e, ASR_E_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes, p->total);
  if (reinterpret_cast<uintptr_t>(ws) & 255) return fail(e, ASR_E_WORKSPACE, "workspace must be 256-byte aligned");
  return ASR_OK;
}

void report_tokens(const Plan& p, const asr_geometry* g, int64_t n, const int64_t* ns, int64_t* out_tokens) {
  if (!out_tokens) return;
  if (ns) {
    for (int b = 0; b < p.B; ++b) out_tokens[b] = p.clips[b].tokens;
  } else {
    *out_tokens = tokens_per_clip(g, n);
  }
}

// A uniform forward through the graph cache: replay when the pointers and
// shape match the recorded forward, else record it (stream capture on the
// encoder's own stream) and launch the new graph on `st`.  Variable-length
// batches, profiling and a failed capture take the direct path.
asr_status run_forward_cached(asr_enc* e, const float* pcm, const Plan& p, float* out, char* ws, cudaStream_t st) {
  // a caller recording its own graph on `st` records the kernels directly
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) {
    (void)cudaGetLastError();
    cs = cudaStreamCaptureStatusActive;
  }
  if (!e->graphs || e->prof || p.varlen || cs != cudaStreamCaptureStatusNone) return run_forward(e, pcm, p, out, ws, st);
  asr_enc::GraphKey key;
  key.pcm = pcm;
  key.out = out;
  key.ws = ws;
  key.n = p.n;
  key.B = p.B;
  key.taps = e->taps;
  if (!e->gexec || !(key == e->gkey)) {
    if (e->gexec) {
      cudaGraphExecDestroy(e->gexec);
      e->gexec = nullptr;
    }
    if (!e->cap_st && cudaStreamCreateWithFlags(&e->cap_st, cudaStreamNonBlocking) != cudaSuccess) {
      e->cap_st = nullptr;
      e->graphs = false;
      (void)cudaGetLastError();
      return run_forward(e, pcm, p, out, ws, st);
    }
    cudaGraph_t graph = nullptr;
    bool ok = cudaStreamBeginCapture(e->cap_st, cudaStreamCaptureModeThreadLocal) == cudaSuccess;
    const asr_status r = ok ? run_forward(e, pcm, p, out, ws, e->cap_st) : ASR_E_CUDA;
    if (ok) ok = cudaStreamEndCapture(e->cap_st, &graph) == cudaSuccess && r == ASR_OK;
    if (ok) ok = cudaGraphInstantiate(&e->gexec, graph, 0) == cudaSuccess;
    if (graph) cudaGraphDestroy(graph);
    if (!ok) {
      if (e->gexec) cudaGraphExecDestroy(e->gexec);
      e->gexec = nullptr;
      e->graphs = false;
      (void)cudaGetLastError();
      return run_forward(e, pcm, p, out, ws, st);
    }
    e->gkey = key;
    e->glaunches = e->launches;
  }
  ASR_CUDA(e, cudaGraphLaunch(e->gexec, st));
  e->launches = e->glaunches;
  return ASR_OK;
}

asr_status forward_common(asr_enc* e, const float* pcm, const int64_t* ns, int64_t n, int B, float* out,
                          int64_t* out_tokens, void* workspace, size_t ws_bytes, void* stream) {
  Plan p;
  ASR_TRY(check_forward_args(e, ns, n, B, pcm, out, workspace, ws_bytes, &p));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ASR_TRY(run_forward_cached(e, pcm, p, out, static_cast<char*>(workspace), st));
  e->last_stream = st;
  e->have_last = true;
  e->last_plan = p;
  e->last_ws = workspace;
  report_tokens(p, &e->g, n, ns, out_tokens);
  return ASR_OK;
}

asr_status forward_host_common(asr_enc* e, const float* pcm_host, const int64_t* ns, int64_t n, int B, float* out_host,
                               int64_t* out_tokens, void* workspace, size_t ws_bytes, void* stream) {
  Plan p;
  ASR_TRY(check_forward_args(e, ns, n, B, pcm_host, out_host, workspace, ws_bytes, &p));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  float* dpcm = reinterpret_cast<float*>(ws + p.off_pcm);
  ASR_CUDA(e, cudaMemcpyAsync(dpcm, pcm_host, (size_t)p.n_total * 4, cudaMemcpyHostToDevice, st));
  const size_t out_bytes = (size_t)p.T * d_out(&e->g) * 4;
  float* dout = reinterpret_cast<float*>(ws + p.off_out);
  ASR_TRY(run_forward_cached(e, dpcm, p, dout, ws, st));
  ASR_CUDA(e, cudaMemcpyAsync(out_host, dout, out_bytes, cudaMemcpyDeviceToHost, st));
  e->last_stream = st;
  e->have_last = true;
  e->last_plan = p;
  e->last_ws = workspace;
  report_tokens(p, &e->g, n, ns, out_tokens);
  return asr_enc_sync_status(e);
}

}  // namespace

extern "C" {

size_t asr_enc_workspace_size(const asr_enc* e, int64_t n_samples, int batch) {
  Plan p;
  if (!e || !plan_for(e, nullptr, n_samples, batch, &p)) return 0;
  return p.total;
}

size_t asr_enc_workspace_size_varlen(const asr_enc* e, const int64_t* n_samples, int batch) {
  Plan p;
  if (!e || !n_samples || !plan_for(e, n_samples, 0, batch, &p)) return 0;
  return p.total;
}

asr_status asr_enc_forward(asr_enc* e, const float* pcm, int64_t n_samples, int batch, float* out, int64_t* out_tokens,
                           void* workspace, size_t ws_bytes, void* stream) {
  return forward_common(e, pcm, nullptr, n_samples, batch, out, out_tokens, workspace, ws_bytes, stream);
}

asr_status asr_enc_forward_varlen(asr_enc* e, const float* pcm, const int64_t* n_samples, int batch, float* out,
                                  int64_t* out_tokens, void* workspace, size_t ws_bytes, void* stream) {
  if (!n_samples) return fail(e, ASR_E_INVAL, "n_samples is NULL");
  return forward_common(e, pcm, n_samples, 0, batch, out, out_tokens, workspace, ws_bytes, stream);
}

asr_status asr_enc_sync_status(asr_enc* e) {
  if (!e) return fail(nullptr, ASR_E_INVAL, "handle is NULL");
  cudaStream_t st = e->have_last ? e->last_stream : nullptr;
  ASR_CUDA(e, cudaStreamSynchronize(st));
  int s = 0;
  ASR_CUDA(e, cudaMemcpy(&s, e->status, 4, cudaMemcpyDeviceToHost));
  if (s != 0) return fail(e, ASR_E_DEVICE_TIMEOUT, "a bounded device wait gave up (code %d)", s);
  return ASR_OK;
}

asr_status asr_enc_forward_host(asr_enc* e, const float* pcm_host, int64_t n_samples, int batch, float* out_host,
                                int64_t* out_tokens, void* workspace, size_t ws_bytes, void* stream) {
  return forward_host_common(e, pcm_host, nullptr, n_samples, batch, out_host, out_tokens, workspace, ws_bytes, stream);
}

asr_status asr_enc_forward_host_varlen(asr_enc* e, const float* pcm_host, const int64_t* n_samples, int batch,
                                       float* out_host, int64_t* out_tokens, void* workspace, size_t ws_bytes,
                                       void* stream) {
  if (!n_samples) return fail(e, ASR_E_INVAL, "n_samples is NULL");
  return forward_host_common(e, pcm_host, n_samples, 0, batch, out_host, out_tokens, workspace, ws_bytes, stream);
}

asr_status asr_enc_set_taps(asr_enc* e, unsigned mask) {
  if (!e) return fail(nullptr, ASR_E_INVAL, "handle is NULL");
  if (mask >> ASR_TAP_COUNT) return fail(e, ASR_E_INVAL, "unknown tap bits");
  e->taps = mask;
  e->maps.ws = nullptr;
  return ASR_OK;
}

asr_status asr_enc_tap(asr_enc* e, int stage, float* dst, size_t dst_bytes, void* stream) {
  if (!e) return fail(nullptr, ASR_E_INVAL, "handle is NULL");
  if (stage < 0 || stage >= ASR_TAP_COUNT) return fail(e, ASR_E_INVAL, "unknown tap stage %d", stage);
  if (!((e->taps >> stage) & 1u) || !e->have_last) return fail(e, ASR_E_INVAL, "tap %d not recorded", stage);
  const size_t bytes = e->last_plan.tap_bytes[stage];
  if (!dst || dst_bytes < bytes) return fail(e, ASR_E_INVAL, "tap needs %zu bytes", bytes);
  ASR_CUDA(e, cudaMemcpyAsync(dst, static_cast<char*>(e->last_ws) + e->last_plan.off_tap[stage], bytes,
                              cudaMemcpyDeviceToDevice, static_cast<cudaStream_t>(stream)));
  return ASR_OK;
}

asr_status asr_enc_set_graphs(asr_enc* e, int enable) {
  if (!e) return fail(nullptr, ASR_E_INVAL, "handle is NULL");
  e->graphs = enable != 0;
  if (!e->graphs && e->gexec) {
    cudaGraphExecDestroy(e->gexec);
    e->gexec = nullptr;
  }
  return ASR_OK;
}

asr_status asr_enc_set_ln_fusion(asr_enc* e, int enable) {
  if (!e) return fail(nullptr, ASR_E_INVAL, "handle is NULL");
  e->ln_fuse_on = enable != 0;
  if (e->gexec) {  // the recorded forward has the other kernel sequence
    cudaGraphExecDestroy(e->gexec);
    e->gexec = nullptr;
  }
  return ASR_OK;
}

asr_status asr_enc_ln_fusion(const asr_enc* e, int* active) {
  if (!e || !active) return fail(nullptr, ASR_E_INVAL, "handle or output is NULL");
  *active = (e->ln_fuse && e->ln_fuse_on) ? 1 : 0;
  return ASR_OK;
}

asr_status asr_enc_profile(asr_enc* e, int enable) {
  if (!e) return fail(nullptr, ASR_E_INVAL, "handle is NULL");
  e->prof = enable != 0;
  return ASR_OK;
}

int asr_enc_profile_read(asr_enc* e, int max, const char** names, double* ms, int* launches) {
  if (!e || max < 0) return -1;
  if (!e->have_last) return 0;
  if (cudaStreamSynchronize(e->last_stream) != cudaSuccess) return -1;
  double tot[PC_COUNT] = {0};
  int cnt[PC_COUNT] = {0};
  for (auto& r : e->prof_recs) {
    float t = 0.f;
    if (cudaEventElapsedTime(&t, e->ev_pool[r.second], e->ev_pool[r.second + 1]) != cudaSuccess) return -1;
    tot[r.first] += t;
    cnt[r.first] += 1;
  }
  int k = 0;
  for (int c = 0; c < PC_COUNT && k < max; ++c) {
    if (!cnt[c]) continue;
    if (names) names[k] = kProfNames[c];
    if (ms) ms[k] = tot[c];
    if (launches) launches[k] = cnt[c];
    ++k;
  }
  return k;
}

int asr_enc_last_launches(const asr_enc* e) { return e ? e->launches : -1; }

// ==================================================================== ops

// Log-mel workspace: [clip maxima (256-byte aligned)][tables].
static size_t log_mel_max_bytes(int batch) { return align_up((size_t)batch * 4, 256); }
size_t asr_op_log_mel_ws_size(int batch) {
  return batch > 0 ? log_mel_max_bytes(batch) + align_up(sizeof(MelTables), 256) : 0;
}

asr_status asr_op_log_mel(const float* pcm, int64_t n_samples, int batch, int n_mels, float* mel, void* ws,
                          size_t ws_bytes, void* stream) {
  if (!pcm || !mel || batch <= 0 || n_mels <= 0 || n_mels > 128 || n_samples <= 200 || n_samples % 160)
    return fail(nullptr, ASR_E_INVAL, "log_mel: bad arguments");
  if (!ws || ws_bytes < asr_op_log_mel_ws_size(batch)) return fail(nullptr, ASR_E_WORKSPACE, "log_mel: workspace too small");
  if (reinterpret_cast<uintptr_t>(ws) & 255) return fail(nullptr, ASR_E_WORKSPACE, "log_mel: workspace must be 256-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned* cm = static_cast<unsigned*>(ws);
  MelTables* tab = reinterpret_cast<MelTables*>(static_cast<char*>(ws) + log_mel_max_bytes(batch));
  ASR_CUDA(nullptr, launch_mel_tables(n_mels, tab, st));
  ASR_CUDA(nullptr, cudaMemsetAsync(cm, 0, (size_t)batch * 4, st));
  ASR_CUDA(nullptr, launch_log_mel(pcm, n_samples, batch, n_mels, tab, mel, cm, st));
  ASR_CUDA(nullptr, launch_mel_normalize(mel, cm, (long long)n_mels * (n_samples / 160), batch, mel, st));
  return ASR_OK;
}

// Device SM count of the current device (the GEMM grid and stream-K scratch size).
static int current_sm_count() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}
// Linear-op workspace: [status word, 256 B][stream-K flags].
static size_t linear_flags_bytes(int sms) { return ((size_t)sms * 8 * 4 + 255) / 256 * 256; }
size_t asr_op_linear_ws_size(void) { return 256 + linear_flags_bytes(current_sm_count()); }

asr_status asr_op_linear(const void* x, const void* w, const float* bias, int64_t M, int N, int K, int epi,
                         int tile_n, void* y, void* ws, size_t ws_bytes, void* stream) {
  if (!x || !w || !y || M <= 0 || N <= 0 || K <= 0 || K % 8 || N % 16)
    return fail(nullptr, ASR_E_INVAL, "linear: bad arguments (K %% 8, N %% 16)");
  if (!ws || ws_bytes < 256) return fail(nullptr, ASR_E_WORKSPACE, "linear: workspace too small");
  int e_bits;
  switch (epi) {
    case ASR_EPI_BF16: e_bits = 0; break;
    case ASR_EPI_BF16_GELU: e_bits = EPI_GELU; break;
    case ASR_EPI_F32_RESID: e_bits = EPI_RESID; break;
    case ASR_EPI_F32: e_bits = EPI_OUT_F32; break;
    case ASR_EPI_SWIGLU:
      if (N % 32) return fail(nullptr, ASR_E_INVAL, "linear: SwiGLU needs N %% 32 == 0");
      e_bits = EPI_SWIGLU;
      break;
    default: return fail(nullptr, ASR_E_INVAL, "linear: unknown epilogue %d", epi);
  }
  const int sms = current_sm_count();
  GemmB wb;
  wb.ptr = static_cast<const bf16*>(w);
  wb.N = N;
  wb.K = K;
  CUtensorMap amap;
  if (!make_weight_maps(wb) || !make_tmap_bf16(&amap, x, M, K, K, 128))
    return fail(nullptr, ASR_E_INVAL, "linear: TMA descriptor encoding failed (16-byte alignment?)");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  GemmParams p;
  memset(&p, 0, sizeof p);
  p.M = (int)M;
  p.out = y;
  p.ldo = (e_bits & EPI_SWIGLU) ? N / 2 : N;
  p.bias = bias;
  p.pe_period = 1;
  p.status = static_cast<int*>(ws);
  p.limit_ns = kWaitLimitNs;
  const size_t fb = linear_flags_bytes(sms);
  if (ws_bytes >= 256 + fb) {
    // Enough scratch for stream-K: flags zeroed together with the status word.
    p.sk_flags = reinterpret_cast<int*>(static_cast<char*>(ws) + 256);
    ASR_CUDA(nullptr, cudaMemsetAsync(ws, 0, 256 + fb, st));
  } else {
    ASR_CUDA(nullptr, cudaMemsetAsync(ws, 0, 4, st));
  }
  if (tile_n && tile_n != 256 && tile_n != 160 && tile_n != 128 && tile_n != 64 && tile_n != -256 && tile_n != -128)
    return fail(nullptr, ASR_E_INVAL, "linear: tile_n must be 0, 256, 160, 128, 64, -256 or -128");
  if (tile_n == 160 && N % 160) return fail(nullptr, ASR_E_INVAL, "linear: tile_n 160 needs N %% 160 == 0");
  const int bn = tile_n ? tile_n : gemm_pick_bn((int)M, N, sms, false);
  CUtensorMap omap, amap3;
  const bool f32_out = (e_bits & (EPI_OUT_F32 | EPI_RESID)) != 0;
  const bool have_omap = !(e_bits & EPI_SWIGLU) && make_tmap_out(&omap, y, M, N, N, f32_out);
  const bool have_a3 = K % 128 == 0 && make_tmap_3d16(&amap3, x, M, K, K, 128, KIND_BF16);
  ASR_CUDA(nullptr, launch_gemm(&amap, wb, p, e_bits, bn, sms, st, have_omap ? &omap : nullptr, have_a3 ? &amap3 : nullptr));
  return ASR_OK;
}

size_t asr_op_linear_resid_ln_ws_size(int64_t M, int N) {
  if (M <= 0 || N <= 0) return 0;
  const size_t cnt = ((size_t)(M + 31) / 32 * 4 + 255) / 256 * 256;
  return 256 + cnt + (size_t)M * 2 * ((N + 255) / 256) * 16;
}

asr_status asr_op_linear_resid_ln(const void* x, const void* w, const float* bias, const float* gamma,
                                  const float* beta, float eps, int64_t M, int N, int K, float* y, void* h,
                                  void* ws, size_t ws_bytes, void* stream) {
  if (!x || !w || !y || !h || !gamma || !beta || M <= 0 || N <= 0 || K <= 0 || !(eps > 0.f) || M > INT_MAX)
    return fail(nullptr, ASR_E_INVAL, "linear_resid_ln: bad arguments");
  if (K % 128 || N % 32) return fail(nullptr, ASR_E_UNSUPPORTED, "linear_resid_ln: needs K %% 128 == 0 and N %% 32 == 0");
  if (!ws || ws_bytes < asr_op_linear_resid_ln_ws_size(M, N))
    return fail(nullptr, ASR_E_WORKSPACE, "linear_resid_ln: workspace too small");
  const int sms = current_sm_count();
  GemmB wb;
  wb.ptr = static_cast<const bf16*>(w);
  wb.N = N;
  wb.K = K;
  CUtensorMap amap, amap3;
  if ((reinterpret_cast<uintptr_t>(y) | reinterpret_cast<uintptr_t>(h) | reinterpret_cast<uintptr_t>(gamma) |
       reinterpret_cast<uintptr_t>(beta)) & 15)
    return fail(nullptr, ASR_E_INVAL, "linear_resid_ln: y, h, gamma and beta must be 16-byte aligned");
  if (!make_weight_maps(wb) || !make_tmap_bf16(&amap, x, M, K, K, 128) ||
      !make_tmap_3d16(&amap3, x, M, K, K, 128, KIND_BF16))
    return fail(nullptr, ASR_E_INVAL, "linear_resid_ln: TMA descriptor encoding failed (16-byte alignment?)");
  if (!gemm_ln_supported(wb, sms)) return fail(nullptr, ASR_E_UNSUPPORTED, "linear_resid_ln: N = %d too wide", N);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t cnt = ((size_t)(M + 31) / 32 * 4 + 255) / 256 * 256;
  ASR_CUDA(nullptr, cudaMemsetAsync(ws, 0, 256 + cnt, st));
  GemmParams p;
  memset(&p, 0, sizeof p);
  p.M = (int)M;
  p.out = y;
  p.ldo = N;
  p.bias = bias;
  p.pe_period = 1;
  p.status = static_cast<int*>(ws);
  p.limit_ns = kWaitLimitNs;
  p.ln_gamma = gamma;
  p.ln_beta = beta;
  p.ln_eps = eps;
  p.ln_count = reinterpret_cast<int*>(static_cast<char*>(ws) + 256);
  p.ln_part = reinterpret_cast<float*>(static_cast<char*>(ws) + 256 + cnt);
  p.ln_h = h;
  p.ln_epoch = 0;  // counters cleared above
  ASR_CUDA(nullptr, launch_gemm(&amap, wb, p, EPI_RESID | EPI_LN, -256, sms, st, nullptr, &amap3));
  return ASR_OK;
}

asr_status asr_op_linear_tf32(const float* x, const float* w, const float* bias, int64_t M, int N, int K, int epi,
                              int tile_n, float* y, void* ws, size_t ws_bytes, void* stream) {
  if (!x || !w || !y || M <= 0 || N <= 0 || K <= 0 || K % 4 || N % 16)
    return fail(nullptr, ASR_E_INVAL, "linear_tf32: bad arguments (K %% 4, N %% 16)");
  if (!ws || ws_bytes < 256) return fail(nullptr, ASR_E_WORKSPACE, "linear_tf32: workspace too small");
  int e_bits;
  switch (epi) {
    case ASR_EPI_F32: e_bits = EPI_OUT_F32; break;
    case ASR_EPI_BF16_GELU: e_bits = EPI_OUT_F32 | EPI_GELU; break;
    case ASR_EPI_F32_RESID: e_bits = EPI_RESID; break;
    case ASR_EPI_SWIGLU:
      if (N % 32) return fail(nullptr, ASR_E_INVAL, "linear_tf32: SwiGLU needs N %% 32 == 0");
      e_bits = EPI_OUT_F32 | EPI_SWIGLU;
      break;
    default: return fail(nullptr, ASR_E_INVAL, "linear_tf32: unsupported epilogue %d", epi);
  }
  if (tile_n && tile_n != 256 && tile_n != 128 && tile_n != 64)
    return fail(nullptr, ASR_E_INVAL, "linear_tf32: tile_n must be 0, 256, 128 or 64");
  const int sms = current_sm_count();
  GemmB wb;
  wb.ptr = w;
  wb.N = N;
  wb.K = K;
  wb.kind = KIND_TF32;
  CUtensorMap amap;
  if (!make_weight_maps(wb) || !make_tmap_f32(&amap, x, M, K, K, 128))
    return fail(nullptr, ASR_E_INVAL, "linear_tf32: TMA descriptor encoding failed (16-byte alignment?)");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  GemmParams p;
  memset(&p, 0, sizeof p);
  p.M = (int)M;
  p.out = y;
  p.ldo = (e_bits & EPI_SWIGLU) ? N / 2 : N;
  p.bias = bias;
  p.pe_period = 1;
  p.status = static_cast<int*>(ws);
  p.limit_ns = kWaitLimitNs;
  ASR_CUDA(nullptr, cudaMemsetAsync(ws, 0, 4, st));
  const int bn = tile_n ? tile_n : gemm_pick_bn_tf32((int)M, N, sms);
  CUtensorMap omap;
  const bool have_omap = !(e_bits & EPI_SWIGLU) && make_tmap_out(&omap, y, M, N, N, true);
  ASR_CUDA(nullptr, launch_gemm(&amap, wb, p, e_bits, bn, sms, st, have_omap ? &omap : nullptr));
  return ASR_OK;
}

asr_status asr_op_layer_norm(const float* x, const float* g, const float* b, int64_t M, int D, float eps, void* y,
                             int out_f32, void* stream) {
  if (!x || !g || !b || !y || M <= 0 || D % 128 || D > 2048) return fail(nullptr, ASR_E_INVAL, "layer_norm: bad arguments");
  ASR_CUDA(nullptr, launch_layer_norm(x, g, b, M, D, eps, y, out_f32 ? KIND_TF32 : KIND_BF16, static_cast<cudaStream_t>(stream)));
  return ASR_OK;
}

size_t asr_op_attention_ws_size(void) { return 256; }

asr_status asr_op_attention(const void* qkv, const int32_t* cu, int n_seg, int max_seg, int64_t T, int H, void* out,
                            void* ws, size_t ws_bytes, void* stream) {
  if (!qkv || !cu || !out || n_seg <= 0 || max_seg <= 0 || H <= 0 || T <= 0)
    return fail(nullptr, ASR_E_INVAL, "attention: bad arguments");
  if (!ws || ws_bytes < 256) return fail(nullptr, ASR_E_WORKSPACE, "attention: workspace too small");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CUtensorMap m;
  if (!make_tmap_qkv(&m, qkv, T, H)) return fail(nullptr, ASR_E_INVAL, "attention: TMA descriptor encoding failed");
  ASR_CUDA(nullptr, cudaMemsetAsync(ws, 0, 4, st));
  if (max_seg <= 128)
    ASR_CUDA(nullptr, launch_attention_tc(m, qkv, cu, n_seg, H, out, static_cast<int*>(ws), kWaitLimitNs, false, st));
  else
    ASR_CUDA(nullptr, launch_attention_fa(m, cu, n_seg, max_seg, H, out, static_cast<int*>(ws), kWaitLimitNs, false, st));
  return ASR_OK;
}

}  // extern "C"

// ---- log-mel entry point that allocates nothing --------------------------
// Its scratch (the per-clip maxima and the FFT / filterbank tables) lives in
// file-scope device arrays that every GPU loading this library holds until
// the process exits.  Host code must not pass these names to a kernel: on
// the host they are stand-ins, not device addresses.  The device addresses
// are looked up once per device (cudaGetSymbolAddress, with that device
// current) and cached here.
namespace {
constexpr int kNoAllocMaxBatch = 4096;  // clips per call
static __device__ __align__(256) unsigned int g_noalloc_clip_max[kNoAllocMaxBatch];
static __device__ __align__(256) MelTables g_noalloc_tables;

struct NoAllocScratch {
  bool ready = false;
  unsigned int* clip_max = nullptr;
  MelTables* tables = nullptr;
};
constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
NoAllocScratch g_noalloc[kNoAllocMaxDevices];
}  // namespace

extern "C" {

asr_status asr_op_log_mel_noalloc(const float* pcm, int64_t n_samples, int batch, int n_mels, float* mel,
                                  void* stream) {
  if (!pcm || !mel || batch <= 0 || n_mels <= 0 || n_mels > 128 || n_samples <= 200 || n_samples % 160)
    return fail(nullptr, ASR_E_INVAL, "log_mel_noalloc: bad arguments");
  if (batch > kNoAllocMaxBatch)
    return fail(nullptr, ASR_E_UNSUPPORTED, "log_mel_noalloc: batch %d exceeds the static scratch limit of %d clips",
                batch, kNoAllocMaxBatch);
  int dev = 0;
  ASR_CUDA(nullptr, cudaGetDevice(&dev));
  if (dev < 0 || dev >= kNoAllocMaxDevices) return fail(nullptr, ASR_E_UNSUPPORTED, "log_mel_noalloc: device %d", dev);
  NoAllocScratch sc;
  {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc[dev].ready) {
      void* cm = nullptr;
      void* tab = nullptr;
      cudaError_t r = cudaGetSymbolAddress(&cm, g_noalloc_clip_max);
      if (r == cudaSuccess) r = cudaGetSymbolAddress(&tab, g_noalloc_tables);
      if (r != cudaSuccess)
        return fail(nullptr, ASR_E_CUDA, "log_mel_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(r));
      g_noalloc[dev].clip_max = static_cast<unsigned int*>(cm);
      g_noalloc[dev].tables = static_cast<MelTables*>(tab);
      g_noalloc[dev].ready = true;
    }
    sc = g_noalloc[dev];
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // Tables are rebuilt on the device and the maxima cleared, in stream order.
  ASR_CUDA(nullptr, launch_mel_tables(n_mels, sc.tables, st));
  ASR_CUDA(nullptr, cudaMemsetAsync(sc.clip_max, 0, (size_t)batch * 4, st));  // the maxima start at zero
  ASR_CUDA(nullptr, launch_log_mel(pcm, n_samples, batch, n_mels, sc.tables, mel, sc.clip_max, st));
  ASR_CUDA(nullptr, launch_mel_normalize(mel, sc.clip_max, (long long)n_mels * (n_samples / 160), batch, mel, st));
  return ASR_OK;
}

size_t asr_splice_ws_size(int64_t n_ids) { return n_ids > 0 ? 256 + align_up((size_t)n_ids * 4, 256) : 0; }

asr_status asr_splice_embeddings(const int32_t* ids, int64_t n_ids, int32_t placeholder, const void* table, int vocab,
                                 int table_dtype, const float* frames, int64_t n_frames, int dim, void* out,
                                 int out_dtype, void* ws, size_t ws_bytes, void* stream) {
  auto dt_ok = [](int d) { return d == ASR_DTYPE_BF16 || d == ASR_DTYPE_F16 || d == ASR_DTYPE_F32; };
  if (!ids || !table || !out || n_ids <= 0 || vocab <= 0 || dim <= 0 || n_frames < 0 || (n_frames > 0 && !frames) ||
      !dt_ok(table_dtype) || !dt_ok(out_dtype) || n_ids > 0x7FFFFFFF)
    return fail(nullptr, ASR_E_INVAL, "splice: bad arguments");
  if (!ws || ws_bytes < asr_splice_ws_size(n_ids) || (reinterpret_cast<uintptr_t>(ws) & 255))
    return fail(nullptr, ASR_E_WORKSPACE, "splice: workspace NULL, unaligned or smaller than asr_splice_ws_size()");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int* status = static_cast<int*>(ws);
  int* rank = reinterpret_cast<int*>(static_cast<char*>(ws) + 256);
  ASR_CUDA(nullptr, cudaMemsetAsync(status, 0, 4, st));
  ASR_CUDA(nullptr, launch_splice(ids, n_ids, placeholder, table, vocab, table_dtype, frames, n_frames, dim, out,
                                  out_dtype, rank, status, current_sm_count(), st));
  return ASR_OK;
}

asr_status asr_splice_check(const void* ws, void* stream) {
  if (!ws) return fail(nullptr, ASR_E_INVAL, "splice_check: ws is NULL");
  ASR_CUDA(nullptr, cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  int s = 0;
  ASR_CUDA(nullptr, cudaMemcpy(&s, ws, 4, cudaMemcpyDeviceToHost));
  if (s == SPLICE_E_ID) return fail(nullptr, ASR_E_INVAL, "splice: a token id is outside [0, vocab)");
  if (s == SPLICE_E_COUNT) return fail(nullptr, ASR_E_INVAL, "splice: the placeholder count differs from the frame count");
  return ASR_OK;
}

asr_status asr_op_gelu(const float* x, float* y, int64_t n, void* stream) {
  if (!x || !y || n <= 0) return fail(nullptr, ASR_E_INVAL, "gelu: bad arguments");
  ASR_CUDA(nullptr, launch_gelu(x, y, n, static_cast<cudaStream_t>(stream)));
  return ASR_OK;
}

asr_status asr_op_wait_probe(int64_t limit_ns, int* status_dev, void* stream) {
  if (!status_dev || limit_ns <= 0 || limit_ns > 10LL * 1000 * 1000 * 1000)
    return fail(nullptr, ASR_E_INVAL, "wait_probe: bad arguments (limit 1 ns .. 10 s)");
  ASR_CUDA(nullptr, launch_wait_probe((unsigned long long)limit_ns, status_dev, static_cast<cudaStream_t>(stream)));
  return ASR_OK;
}


}  // extern "C"

// ---- streaming ------------------------------------------------------------
// A live stream is encoded one attention window at a time (the windows are
// independent: "MOSS-Transcribe-preview-2B-GGUF", Architecture, "Audio
// encoder", windowed block-diagonal attention).  Window j covers the stream's
// mel frames [j WF, (j + 1) WF), WF = window_tokens / tokens-per-chunk *
// chunk_frames (800 frames, 8 s, for 104-token windows of 100-frame chunks).
// Its frames are the centred frames of the whole stream (real samples on
// both sides, reflection only at the stream's start and end), and its log-mel
// is normalised by the maximum over its own frames, so a window can be
// encoded as soon as the samples its last frame reads have arrived:
// ((j + 1) WF - 1) hop + n_fft / 2 of them (128040 for window 0).  Each
// ready window is one clip of a variable-length forward whose samples start
// at the window's first frame centre with n_fft / 2 real samples of history
// before it (none for window 0).
struct asr_stream {
  asr_enc* e = nullptr;
  float* buf[2] = {nullptr, nullptr};
  size_t cap = 0;            // floats per buffer
  int cur = 0;
  int64_t base = 0;          // absolute index of buf[cur][0]
  int64_t len = 0;           // samples held in buf[cur]
  int64_t total = 0;         // samples pushed
  int64_t next_win = 0;      // next window to encode
  int wf = 0;                // frames per window
  int64_t wtok = 0;          // tokens of a whole window
  bool finished = false;
};

namespace {

void stream_free_bufs(asr_stream* s) {
  for (float*& b : s->buf) {
    if (!b) continue;
    if (s->e->free_fn)
      s->e->free_fn(s->e->ctx, b);
    else if (!s->e->alloc)
      cudaFree(b);
    b = nullptr;
  }
}

void* stream_alloc(asr_enc* e, size_t bytes) {
  if (e->alloc) return e->alloc(e->ctx, bytes);
  void* p = nullptr;
  return cudaMalloc(&p, bytes) == cudaSuccess ? p : nullptr;
}

// Stream windows j0 .. j0 + k - 1 (k >= 1; `final` = the last one ends the
// stream) as one variable-length forward writing k windows' rows to `out`.
asr_status stream_encode(asr_stream* s, int64_t j0, int k, bool final, float* out, int64_t out_cap, int64_t* rows,
                         void* ws, size_t ws_bytes, cudaStream_t st) {
  asr_enc* e = s->e;
  const int hop = e->g.hop, half = e->g.n_fft / 2;
  std::vector<int64_t> ns(k), offs(k);
  std::vector<int> lefts(k);
  for (int i = 0; i < k; ++i) {
    // the window's first frame is centred on sample `start`; a whole window's
    // last frame reads up to start + (WF - 1) hop + n_fft / 2 - 1, and that
    // length gives exactly WF frames (hop <= n_fft / 2 < 2 hop)
    const int64_t start = (j0 + i) * s->wf * (int64_t)hop;
    const bool last = final && i == k - 1;
    ns[i] = last ? s->total - start : (int64_t)(s->wf - 1) * hop + half;
    offs[i] = start - s->base;
    lefts[i] = start > 0 ? half : 0;
  }
  Plan p;
  if (!make_plan_varlen(e, ns.data(), k, &p, offs.data(), lefts.data()))
    return fail(e, ASR_E_UNSUPPORTED, "stream: window plan failed");
  if (p.T > out_cap) return fail(e, ASR_E_INVAL, "stream: out holds %lld rows, %lld needed", (long long)out_cap, (long long)p.T);
  if (!ws || ws_bytes < p.total || (reinterpret_cast<uintptr_t>(ws) & 255))
    return fail(e, ASR_E_WORKSPACE, "stream: workspace %zu bytes < %zu needed (or not 256-byte aligned)", ws_bytes, p.total);
  ASR_TRY(run_forward(e, s->buf[s->cur], p, out, static_cast<char*>(ws), st));
  e->last_stream = st;
  e->have_last = true;
  e->last_plan = p;
  e->last_ws = ws;
  *rows = p.T;
  return ASR_OK;
}

}  // namespace

extern "C" {

int64_t asr_stream_window_tokens(const asr_enc* e) {
  if (!e || e->g.stem != ASR_STEM_CONV2D_CHUNKED || !e->g.window_tokens) return -1;
  const int64_t t3 = chunk_tokens(e->g.chunk_frames);
  return e->g.window_tokens % t3 ? -1 : e->g.window_tokens;
}

size_t asr_stream_workspace_size(const asr_enc* e, int windows) {
  if (!e || windows <= 0 || asr_stream_window_tokens(e) <= 0) return 0;
  const int wf = (int)(e->g.window_tokens / chunk_tokens(e->g.chunk_frames)) * e->g.chunk_frames;
  const int half = e->g.n_fft / 2;
  std::vector<int64_t> ns(windows, (int64_t)(wf - 1) * e->g.hop + half), offs(windows, 0);
  std::vector<int> lefts(windows, half);
  Plan p;
  if (!make_plan_varlen(e, ns.data(), windows, &p, offs.data(), lefts.data())) return 0;
  return p.total;
}

asr_status asr_stream_create(asr_enc* e, asr_stream** out) {
  if (!e || !out) return fail(e, ASR_E_INVAL, "stream_create: NULL argument");
  *out = nullptr;
  if (asr_stream_window_tokens(e) <= 0)
    return fail(e, ASR_E_UNSUPPORTED, "streaming needs the chunked conv2d stem and windows of whole chunks");
  asr_stream* s = new asr_stream();
  s->e = e;
  s->wf = (int)(e->g.window_tokens / chunk_tokens(e->g.chunk_frames)) * e->g.chunk_frames;
  s->wtok = e->g.window_tokens;
  *out = s;
  return ASR_OK;
}

void asr_stream_destroy(asr_stream* s) {
  if (!s) return;
  stream_free_bufs(s);
  delete s;
}

asr_status asr_stream_push(asr_stream* s, const float* pcm, int64_t n, float* out, int64_t out_cap_rows,
                           int64_t* out_rows, void* ws, size_t ws_bytes, void* stream) {
  if (!s || !out_rows || n < 0 || (n > 0 && !pcm)) return fail(s ? s->e : nullptr, ASR_E_INVAL, "stream_push: bad arguments");
  asr_enc* e = s->e;
  *out_rows = 0;
  if (s->finished) return fail(e, ASR_E_INVAL, "stream_push: the stream is finished");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int hop = e->g.hop, half = e->g.n_fft / 2;
  // room for the new samples (buffers grow through the encoder's allocator)
  if ((size_t)(s->len + n) > s->cap) {
    size_t cap = std::max<size_t>(s->cap * 2, (size_t)(s->len + n) + (size_t)s->wf * hop);
    float* nb[2] = {static_cast<float*>(stream_alloc(e, cap * 4)), static_cast<float*>(stream_alloc(e, cap * 4))};
    if (!nb[0] || !nb[1]) {
      for (float* b : nb)
        if (b) {
          if (e->free_fn) e->free_fn(e->ctx, b); else if (!e->alloc) cudaFree(b);
        }
      return fail(e, ASR_E_NOMEM, "stream_push: buffer allocation of %zu bytes failed", cap * 4);
    }
    if (s->len) ASR_CUDA(e, cudaMemcpyAsync(nb[0], s->buf[s->cur], (size_t)s->len * 4, cudaMemcpyDeviceToDevice, st));
    // the old buffers may still be read by queued work on `stream`
    ASR_CUDA(e, cudaStreamSynchronize(st));
    stream_free_bufs(s);
    s->buf[0] = nb[0];
    s->buf[1] = nb[1];
    s->cur = 0;
    s->cap = cap;
  }
  if (n) ASR_CUDA(e, cudaMemcpyAsync(s->buf[s->cur] + s->len, pcm, (size_t)n * 4, cudaMemcpyDeviceToDevice, st));
  s->len += n;
  s->total += n;
  // windows whose last frame's samples have all arrived
  int64_t k = 0;
  while ((s->next_win + k + 1) * s->wf * (int64_t)hop - hop + half <= s->total) ++k;
  if (k == 0) return ASR_OK;
  ASR_TRY(stream_encode(s, s->next_win, (int)k, false, out, out_cap_rows, out_rows, ws, ws_bytes, st));
  s->next_win += k;
  // keep n_fft / 2 samples of history before the next window
  const int64_t keep = std::max<int64_t>(0, s->next_win * s->wf * (int64_t)hop - half);
  if (keep > s->base) {
    const int64_t drop = keep - s->base;
    const int nxt = s->cur ^ 1;
    if (s->len - drop > 0)
      ASR_CUDA(e, cudaMemcpyAsync(s->buf[nxt], s->buf[s->cur] + drop, (size_t)(s->len - drop) * 4,
                                  cudaMemcpyDeviceToDevice, st));
    s->cur = nxt;
    s->len -= drop;
    s->base = keep;
  }
  return ASR_OK;
}

asr_status asr_stream_finish(asr_stream* s, float* out, int64_t out_cap_rows, int64_t* out_rows, void* ws,
                             size_t ws_bytes, void* stream) {
  if (!s || !out_rows) return fail(s ? s->e : nullptr, ASR_E_INVAL, "stream_finish: bad arguments");
  asr_enc* e = s->e;
  *out_rows = 0;
  if (s->finished) return fail(e, ASR_E_INVAL, "stream_finish: the stream is finished");
  if (s->total <= e->g.n_fft / 2) return fail(e, ASR_E_INVAL, "stream_finish: a stream needs more than n_fft/2 samples");
  s->finished = true;
  const int64_t frames_left = s->total / e->g.hop - s->next_win * s->wf;
  if (frames_left <= 0) return ASR_OK;
  return stream_encode(s, s->next_win, 1, true, out, out_cap_rows, out_rows, ws, ws_bytes,
                       static_cast<cudaStream_t>(stream));
}

}  // extern "C"
