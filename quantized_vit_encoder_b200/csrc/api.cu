// C ABI of libvitq.so: argument validation, TMA tensor-map encoding, and the
// block / merger / tower drivers that chain the kernels on the caller's stream.
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "internal.h"
#include "vitq.h"

namespace vitq {

static std::atomic<unsigned long long> g_launches{0};

// Optional per-launch timing (vitq_profile_*): a CUDA event pair around every
// kernel launch on the launching stream, plus the launch's algorithmic work.
struct ProfRecord {
  const char* name;
  cudaEvent_t a, b;
  double flops, bytes;
};
static std::mutex g_prof_mu;
static bool g_prof_on = false;
static std::vector<ProfRecord> g_prof;
static std::vector<float> g_prof_ms;

static void prof_begin(const char* name, cudaStream_t st, double flops, double bytes) {
  if (!g_prof_on) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  ProfRecord r{name, nullptr, nullptr, flops, bytes};
  cudaEventCreate(&r.a);
  cudaEventCreate(&r.b);
  cudaEventRecord(r.a, st);
  g_prof.push_back(r);
}
static void prof_end(cudaStream_t st) {
  if (!g_prof_on) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  cudaEventRecord(g_prof.back().b, st);
}

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  int checked = 0;  // 0 unknown, 1 ok, -1 not sm_100
  int num_sms = 0;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

int current_device_ok(int* num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return VITQ_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (d.checked == 0) {
    cudaDeviceProp p;
    if (cudaGetDeviceProperties(&p, dev) != cudaSuccess) return VITQ_ERR_CUDA;
    if (p.major == 10 && p.minor == 0) {
      // one-time setup: the GELU table of this device, built on a private stream
      cudaStream_t s;
      if (cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) != cudaSuccess) return VITQ_ERR_CUDA;
      cudaError_t e = build_gelu_table(s);
      if (e == cudaSuccess) e = cudaStreamSynchronize(s);
      cudaStreamDestroy(s);
      if (e != cudaSuccess) return VITQ_ERR_CUDA;
    }
    d.checked = (p.major == 10 && p.minor == 0) ? 1 : -1;
    d.num_sms = p.multiProcessorCount;
  }
  if (d.checked < 0) return VITQ_ERR_ARCH;
  if (num_sms) *num_sms = d.num_sms;
  return VITQ_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t up256(size_t b) { return (b + 255) & ~size_t(255); }
inline int up4(int v) { return (v + 3) & ~3; }
inline cudaStream_t S(void* s) { return reinterpret_cast<cudaStream_t>(s); }

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return VITQ_OK;
  return VITQ_ERR_CUDA;
}

int pick_block_n(int M, int N, int num_sms) {
  if (const char* env = std::getenv("VITQ_GEMM_BN")) {
    const int v = std::atoi(env);
    if (v == 64 || v == 128 || v == 256) return v;
  }
  // Every 128-wide K block of a tile costs a fixed ~580 cycles of MMA issue
  // whatever the tile width (measured), so 128 x 256 tiles, with half as many K
  // blocks per output, win where N is wide and M fills the GPU; narrow outputs
  // keep 128 for enough tiles per SM (and four TMEM partial buffers, which hide
  // the epilogue).  Where the narrower tiling still leaves half of the SMs free
  // (small M), it runs each tile sooner and on more SMs; a narrower tiling that
  // fills the GPU measured slower in the block (the next kernel, launched early,
  // finds no free SM to start on).  Each output element is computed the same way
  // at every tile width, so the choice does not change results.
  const long long tiles_m = (M + 127) / 128;
  const long long half = num_sms / 2;
  if (N > 1536) return tiles_m * ((N + 127) / 128) <= half ? 128 : 256;
  return tiles_m * ((N + 63) / 64) <= half ? 64 : 128;
}

// Workspace carving helper.
struct Carver {
  uint8_t* p;
  size_t used = 0;
  template <class T>
  T* take(size_t bytes) {
    T* r = reinterpret_cast<T*>(p ? p + used : nullptr);
    used += up256(bytes);
    return r;
  }
};

struct BlockWs {
  uint8_t* q;
  float* s;
  __nv_bfloat16 *qkv, *attn, *x1, *f;
  int lds;
};

BlockWs carve_block(Carver& c, int n) {
  BlockWs w;
  w.lds = up4(n);
  w.q = c.take<uint8_t>((size_t)n * VITQ_MLP);
  w.s = c.take<float>((size_t)((VITQ_MLP + 127) / 128) * w.lds * 4);
  w.qkv = c.take<__nv_bfloat16>((size_t)n * VITQ_QKV * 2);
  w.attn = c.take<__nv_bfloat16>((size_t)n * VITQ_HIDDEN * 2);
  w.x1 = c.take<__nv_bfloat16>((size_t)n * VITQ_HIDDEN * 2);
  w.f = c.take<__nv_bfloat16>((size_t)n * VITQ_MLP * 2);
  return w;
}

struct MergerWs {
  uint8_t* q;
  float* s;
  __nv_bfloat16* h;
  int lds;
};

MergerWs carve_merger(Carver& c, int n_tokens) {
  const int m = n_tokens / 4;
  MergerWs w;
  w.lds = up4(m);
  w.q = c.take<uint8_t>((size_t)m * VITQ_MERGE_IN);
  w.s = c.take<float>((size_t)(VITQ_MERGE_IN / 128) * w.lds * 4);
  w.h = c.take<__nv_bfloat16>((size_t)m * VITQ_MERGE_IN * 2);
  return w;
}

struct MergerBf16Ws {
  __nv_bfloat16 *ln, *h;
};

MergerBf16Ws carve_merger_bf16(Carver& c, int n_tokens) {
  const int m = n_tokens / 4;
  MergerBf16Ws w;
  w.ln = c.take<__nv_bfloat16>((size_t)m * VITQ_MERGE_IN * 2);
  w.h = c.take<__nv_bfloat16>((size_t)m * VITQ_MERGE_IN * 2);
  return w;
}

struct TowerWs {
  int32_t* pos;
  int32_t* cu;
  float* cs;
  uint8_t* rest;
};

TowerWs carve_tower_head(Carver& c, int n, int n_images) {
  TowerWs t;
  t.pos = c.take<int32_t>((size_t)n * 2 * 4);
  t.cu = c.take<int32_t>((size_t)(n_images + 1) * 4);
  t.cs = c.take<float>((size_t)n * 72 * 4);
  return t;
}

// Launch one kernel through `expr`, counting it and (when profiling) timing it.
#define VITQ_LAUNCH(name, st, flops, bytes, expr)    \
  do {                                               \
    prof_begin(name, st, (double)(flops), (double)(bytes)); \
    const cudaError_t e_ = (expr);                   \
    prof_end(st);                                    \
    g_launches.fetch_add(1);                         \
    if (e_ != cudaSuccess) return VITQ_ERR_CUDA;     \
  } while (0)

#define VITQ_CHECK(cond, code) \
  do {                         \
    if (!(cond)) return (code); \
  } while (0)

// CTA pairs (cta_group::2 MMA) for the GEMMs; VITQ_GEMM_PAIR=0 selects one CTA per tile.
bool pick_pair() {
  if (const char* env = std::getenv("VITQ_GEMM_PAIR")) return std::atoi(env) != 0;
  return false;
}

int gemm_checked(const uint8_t* A, const float* sA, int ldsA, const uint8_t* W, const float* sW,
                 const void* bias, const void* residual, void* C, int M, int N, int K, int num_sms,
                 cudaStream_t st) {
  const double mn = (double)M * N;
  VITQ_LAUNCH("fp8_block_gemm", st, 2.0 * mn * K,
              (double)M * K + (double)N * K + mn * 2 * (residual ? 2 : 1) + (double)((K + 127) / 128) * M * 4,
              launch_fp8_gemm(A, sA, ldsA, W, sW, reinterpret_cast<const __nv_bfloat16*>(bias),
                           reinterpret_cast<const __nv_bfloat16*>(residual),
                           reinterpret_cast<__nv_bfloat16*>(C), M, N, K, pick_block_n(M, N, num_sms),
                           pick_pair(), num_sms, st));
  return VITQ_OK;
}

int bf16_gemm_checked(const __nv_bfloat16* A, const __nv_bfloat16* W, const __nv_bfloat16* bias,
                      const __nv_bfloat16* residual, __nv_bfloat16* C, int M, int N, int K, int num_sms,
                      cudaStream_t st) {
  const double mn = (double)M * N;
  VITQ_LAUNCH("bf16_gemm", st, 2.0 * mn * K,
              2.0 * ((double)M * K + (double)N * K) + mn * 2 * (residual ? 2 : 1),
              launch_bf16_gemm(A, W, bias, residual, C, M, N, K, pick_block_n(M, N, num_sms), num_sms, st));
  return VITQ_OK;
}

bool block_weights_ok(const vitq_block_weights* w) {
  return w && w->norm1_w && w->norm1_b && w->qkv_q && w->qkv_s && w->qkv_b && w->proj_q && w->proj_s &&
         w->proj_b && w->norm2_w && w->norm2_b && w->fc1_q && w->fc1_s && w->fc1_b && w->fc2_q &&
         w->fc2_s && w->fc2_b && al16(w->qkv_q) && al16(w->proj_q) && al16(w->fc1_q) && al16(w->fc2_q) &&
         al16(w->qkv_b) && al16(w->proj_b) && al16(w->fc1_b) && al16(w->fc2_b) && al16(w->norm1_w) &&
         al16(w->norm1_b) && al16(w->norm2_w) && al16(w->norm2_b);
}

bool merger_weights_ok(const vitq_merger_weights* w) {
  return w && w->norm_w && w->norm_b && w->fc1_q && w->fc1_s && w->fc1_b && w->fc2_q && w->fc2_s &&
         w->fc2_b && al16(w->fc1_q) && al16(w->fc2_q) && al16(w->fc1_b) && al16(w->fc2_b) &&
         al16(w->norm_w) && al16(w->norm_b);
}

// Softmax scale 1/sqrt(72), the fp32 value nearest to it (1/sqrtf(72.f) is one ulp
// below).
const float kSoftmaxScale = (float)(1.0 / std::sqrt((double)VITQ_HEAD_DIM));

// Algorithmic HBM bytes of the row kernels (read bf16 rows, write codes + scales).
inline double quant_bytes(double M, double K) { return M * K * 2 + M * K + M * ((K + 127) / 128) * 4; }

// One FP8 block in place on x ("Qwen3-VL-8B on RTX 5090", section 3, the per-block
// chain; "spark_model/layers/vision_encoder.rs", ViTBlock): LN1+quant, QKV GEMM + bias,
// rotary (v to fp16), attention, quant, proj GEMM + bias + x, LN2+quant, fc1 GEMM +
// bias, GELU+quant, fc2 GEMM + bias + x1.
int block_impl(const vitq_block_weights* w, __nv_bfloat16* x, int n, const int32_t* cu, int n_seqs,
               int max_seqlen, const float* cs, const BlockWs& b, int num_sms, double attn_sumsq,
               cudaStream_t st) {
  const double eps = 1e-6;
  const double dn = n;
  using bf = __nv_bfloat16;
  VITQ_LAUNCH("ln_quant", st, 0, quant_bytes(dn, VITQ_HIDDEN),
              launch_ln_quant(x, VITQ_HIDDEN, (const bf*)w->norm1_w, (const bf*)w->norm1_b, n, VITQ_HIDDEN, eps,
                              b.q, b.s, b.lds, st));
  int r = gemm_checked(b.q, b.s, b.lds, w->qkv_q, w->qkv_s, w->qkv_b, nullptr, b.qkv, n, VITQ_QKV,
                       VITQ_HIDDEN, num_sms, st);
  if (r) return r;
  VITQ_LAUNCH("rope2d", st, 0, dn * 3456 * 2 * 2 + dn * 72 * 4, launch_rope_apply(b.qkv, n, cs, 1, st));
  VITQ_LAUNCH("attention", st, 4.0 * attn_sumsq * VITQ_HEAD_DIM * VITQ_HEADS, dn * VITQ_QKV * 2 + dn * VITQ_HIDDEN * 2,
              launch_attention(b.qkv, n, cu, n_seqs, max_seqlen, kSoftmaxScale, true, b.attn, st));
  VITQ_LAUNCH("quant_act", st, 0, quant_bytes(dn, VITQ_HIDDEN),
              launch_quant_act(b.attn, n, VITQ_HIDDEN, VITQ_HIDDEN, b.q, b.s, b.lds, st));
  r = gemm_checked(b.q, b.s, b.lds, w->proj_q, w->proj_s, w->proj_b, x, b.x1, n, VITQ_HIDDEN, VITQ_HIDDEN,
                   num_sms, st);
  if (r) return r;
  VITQ_LAUNCH("ln_quant", st, 0, quant_bytes(dn, VITQ_HIDDEN),
              launch_ln_quant(b.x1, VITQ_HIDDEN, (const bf*)w->norm2_w, (const bf*)w->norm2_b, n, VITQ_HIDDEN, eps,
                              b.q, b.s, b.lds, st));
  r = gemm_checked(b.q, b.s, b.lds, w->fc1_q, w->fc1_s, w->fc1_b, nullptr, b.f, n, VITQ_MLP, VITQ_HIDDEN,
                   num_sms, st);
  if (r) return r;
  VITQ_LAUNCH("gelu_quant", st, 0, quant_bytes(dn, VITQ_MLP),
              launch_gelu_quant(b.f, n, VITQ_MLP, VITQ_MLP, b.q, b.s, b.lds, num_sms, st));
  return gemm_checked(b.q, b.s, b.lds, w->fc2_q, w->fc2_s, w->fc2_b, b.x1, x, n, VITQ_HIDDEN, VITQ_MLP,
                      num_sms, st);
}

// One FP8 2x2 merger ("Qwen3-VL-8B on RTX 5090", section 3; vision_encoder.rs,
// MergerLayer): four consecutive rows read as one 4608 row, LN+quant, fc1 + bias,
// GELU+quant, fc2 + bias.
int merger_impl(const vitq_merger_weights* w, const __nv_bfloat16* x, int n, __nv_bfloat16* out,
                const MergerWs& m, int num_sms, cudaStream_t st) {
  using bf = __nv_bfloat16;
  const int rows = n / 4;
  VITQ_LAUNCH("ln_quant", st, 0, quant_bytes(rows, VITQ_MERGE_IN),
              launch_ln_quant(x, VITQ_MERGE_IN, (const bf*)w->norm_w, (const bf*)w->norm_b, rows, VITQ_MERGE_IN,
                              1e-6, m.q, m.s, m.lds, st));
  int r = gemm_checked(m.q, m.s, m.lds, w->fc1_q, w->fc1_s, w->fc1_b, nullptr, m.h, rows, VITQ_MERGE_IN,
                       VITQ_MERGE_IN, num_sms, st);
  if (r) return r;
  VITQ_LAUNCH("gelu_quant", st, 0, quant_bytes(rows, VITQ_MERGE_IN),
              launch_gelu_quant(m.h, rows, VITQ_MERGE_IN, VITQ_MERGE_IN, m.q, m.s, m.lds, num_sms, st));
  return gemm_checked(m.q, m.s, m.lds, w->fc2_q, w->fc2_s, w->fc2_b, nullptr, out, rows, VITQ_OUT_HIDDEN,
                      VITQ_MERGE_IN, num_sms, st);
}

bool block_bf16_weights_ok(const vitq_block_weights_bf16* w) {
  const void* p[12] = {w ? w->norm1_w : nullptr, w ? w->norm1_b : nullptr, w ? w->qkv_w : nullptr,
                       w ? w->qkv_b : nullptr,   w ? w->proj_w : nullptr,  w ? w->proj_b : nullptr,
                       w ? w->norm2_w : nullptr, w ? w->norm2_b : nullptr, w ? w->fc1_w : nullptr,
                       w ? w->fc1_b : nullptr,   w ? w->fc2_w : nullptr,   w ? w->fc2_b : nullptr};
  for (const void* q : p)
    if (!q || !al16(q)) return false;
  return true;
}

bool merger_bf16_weights_ok(const vitq_merger_weights_bf16* w) {
  const void* p[6] = {w ? w->norm_w : nullptr, w ? w->norm_b : nullptr, w ? w->fc1_w : nullptr,
                      w ? w->fc1_b : nullptr,  w ? w->fc2_w : nullptr,  w ? w->fc2_b : nullptr};
  for (const void* q : p)
    if (!q || !al16(q)) return false;
  return true;
}

// bf16 block ("Qwen3-VL-8B on RTX 5090", section 4: the first three blocks keep
// bf16): the LayerNorm outputs go to the codes region of the block
// workspace (n * 4304 bytes >= n * 1152 bf16), GELU runs in place on the fc1 output.
int block_bf16_impl(const vitq_block_weights_bf16* w, __nv_bfloat16* x, int n, const int32_t* cu, int n_seqs,
                    int max_seqlen, const float* cs, const BlockWs& b, int num_sms, double attn_sumsq,
                    cudaStream_t st) {
  using bf = __nv_bfloat16;
  const double eps = 1e-6, dn = n;
  bf* h = reinterpret_cast<bf*>(b.q);
  const double ln_bytes = dn * VITQ_HIDDEN * 4;
  VITQ_LAUNCH("ln_bf16", st, 0, ln_bytes,
              launch_ln(x, VITQ_HIDDEN, (const bf*)w->norm1_w, (const bf*)w->norm1_b, n, VITQ_HIDDEN, eps, nullptr,
                        nullptr, 0, h, st));
  int r = bf16_gemm_checked(h, (const bf*)w->qkv_w, (const bf*)w->qkv_b, nullptr, b.qkv, n, VITQ_QKV,
                            VITQ_HIDDEN, num_sms, st);
  if (r) return r;
  VITQ_LAUNCH("rope2d", st, 0, dn * 3456 * 2 * 2 + dn * 72 * 4, launch_rope_apply(b.qkv, n, cs, 1, st));
  VITQ_LAUNCH("attention", st, 4.0 * attn_sumsq * VITQ_HEAD_DIM * VITQ_HEADS, dn * VITQ_QKV * 2 + dn * VITQ_HIDDEN * 2,
              launch_attention(b.qkv, n, cu, n_seqs, max_seqlen, kSoftmaxScale, true, b.attn, st));
  r = bf16_gemm_checked(b.attn, (const bf*)w->proj_w, (const bf*)w->proj_b, x, b.x1, n, VITQ_HIDDEN, VITQ_HIDDEN,
                        num_sms, st);
  if (r) return r;
  VITQ_LAUNCH("ln_bf16", st, 0, ln_bytes,
              launch_ln(b.x1, VITQ_HIDDEN, (const bf*)w->norm2_w, (const bf*)w->norm2_b, n, VITQ_HIDDEN, eps,
                        nullptr, nullptr, 0, h, st));
  r = bf16_gemm_checked(h, (const bf*)w->fc1_w, (const bf*)w->fc1_b, nullptr, b.f, n, VITQ_MLP, VITQ_HIDDEN,
                        num_sms, st);
  if (r) return r;
  VITQ_LAUNCH("gelu_bf16", st, 0, dn * VITQ_MLP * 4,
              launch_gelu(b.f, n, VITQ_MLP, VITQ_MLP, nullptr, nullptr, 0, b.f, num_sms, st));
  return bf16_gemm_checked(b.f, (const bf*)w->fc2_w, (const bf*)w->fc2_b, b.x1, x, n, VITQ_HIDDEN, VITQ_MLP,
                           num_sms, st);
}

// bf16 2x2 merger ("Qwen3-VL-8B on RTX 5090", section 4: the mergers keep bf16).
int merger_bf16_impl(const vitq_merger_weights_bf16* w, const __nv_bfloat16* x, int n, __nv_bfloat16* out,
                     const MergerBf16Ws& m, int num_sms, cudaStream_t st) {
  using bf = __nv_bfloat16;
  const int rows = n / 4;
  VITQ_LAUNCH("ln_bf16", st, 0, (double)rows * VITQ_MERGE_IN * 4,
              launch_ln(x, VITQ_MERGE_IN, (const bf*)w->norm_w, (const bf*)w->norm_b, rows, VITQ_MERGE_IN, 1e-6,
                        nullptr, nullptr, 0, m.ln, st));
  int r = bf16_gemm_checked(m.ln, (const bf*)w->fc1_w, (const bf*)w->fc1_b, nullptr, m.h, rows, VITQ_MERGE_IN,
                            VITQ_MERGE_IN, num_sms, st);
  if (r) return r;
  VITQ_LAUNCH("gelu_bf16", st, 0, (double)rows * VITQ_MERGE_IN * 4,
              launch_gelu(m.h, rows, VITQ_MERGE_IN, VITQ_MERGE_IN, nullptr, nullptr, 0, m.h, num_sms, st));
  return bf16_gemm_checked(m.h, (const bf*)w->fc2_w, (const bf*)w->fc2_b, nullptr, out, rows, VITQ_OUT_HIDDEN,
                           VITQ_MERGE_IN, num_sms, st);
}

}  // namespace

cudaError_t encode_tma_2d_u8(CUtensorMap* tm, const void* base, int cols, int rows, int box_cols,
                             int box_rows) {
  auto enc = get_encode();
  if (!enc) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t encode_tma_2d_bf16(CUtensorMap* tm, const void* base, int cols, int rows, int box_cols,
                               int box_rows) {
  auto enc = get_encode();
  if (!enc) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t encode_tma_qkv(CUtensorMap* tm, const void* qkv, int n_tokens, int box_d, bool lo) {
  auto enc = get_encode();
  if (!enc) return cudaErrorNotSupported;
  cuuint64_t dims[3] = {72, 48, (cuuint64_t)n_tokens};
  cuuint64_t strides[2] = {72 * 2, 3456 * 2};
  cuuint32_t box[3] = {(cuuint32_t)box_d, 1, 128};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(qkv), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, lo ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_32B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace vitq

using namespace vitq;

extern "C" {

int vit_quant_act(const void* x, int M, int K, int ldx, uint8_t* q, float* s, int lds, void* stream) {
  VITQ_CHECK(x && q && s, VITQ_ERR_INVALID_ARG);
  VITQ_CHECK(M >= 0 && K > 0 && ldx >= K && lds >= M, VITQ_ERR_INVALID_ARG);
  VITQ_CHECK(K % 16 == 0 && K <= 4608 && ldx % 8 == 0 && M <= VITQ_MAX_ROWS, VITQ_ERR_SHAPE);
  VITQ_CHECK(al16(x) && al16(q), VITQ_ERR_ALIGN);
  int r = current_device_ok(nullptr);
  if (r) return r;
  VITQ_LAUNCH("quant_act", S(stream), 0, quant_bytes(M, K), launch_quant_act((const __nv_bfloat16*)x, M, K, ldx, q, s, lds, S(stream)));
  return VITQ_OK;
}

int vit_quant_weight(const void* w, int N, int K, uint8_t* q, float* s, void* stream) {
  VITQ_CHECK(w && q && s, VITQ_ERR_INVALID_ARG);
  VITQ_CHECK(N >= 0 && K > 0, VITQ_ERR_INVALID_ARG);
  VITQ_CHECK(K % 16 == 0 && N <= VITQ_MAX_DIM && K <= VITQ_MAX_DIM, VITQ_ERR_SHAPE);
  VITQ_CHECK(al16(w) && al16(q), VITQ_ERR_ALIGN);
  int r = current_device_ok(nullptr);
  if (r) return r;
  VITQ_LAUNCH("quant_weight", S(stream), 0, (double)N * K * 3, launch_quant_weight((const __nv_bfloat16*)w, N, K, q, s, S(stream)));
  return VITQ_OK;
}

int vit_ln_quant(const void* x, int M, int K, int ldx, const void* gamma, const void* beta, float eps,
                 uint8_t* q, float* s, int lds, void* stream) {
  VITQ_CHECK(x && gamma && beta && q && s, VITQ_ERR_INVALID_ARG);
  VITQ_CHECK(M >= 0 && K > 0 && ldx >= K && lds >= M && eps >= 0.f, VITQ_ERR_INVALID_ARG);
  VITQ_CHECK(K % 16 == 0 && K <= 4608 && ldx % 8 == 0 && M <= VITQ_MAX_ROWS, VITQ_ERR_SHAPE);
  VITQ_CHECK(al16(x) && al16(q) && al16(gamma) && al16(beta), VITQ_ERR_ALIGN);
  int r = current_device_ok(nullptr);
  if (r) return r;
  VITQ_LAUNCH("ln_quant", S(stream), 0, quant_bytes(M, K), launch_ln_quant((const __nv_bfloat16*)x, ldx, (const __nv_bfloat16*)gamma,
                           (const __nv_bfloat16*)beta, M, K, (double)eps, q, s, lds, S(stream)));
  return VITQ_OK;
}

int vit_gelu_quant(const void* f, int M, int K, int ldf, uint8_t* q, float* s, int lds, void* stream) {
  VITQ_CHECK(f && q && s, VITQ_ERR_INVALID_ARG);
  VITQ_CHECK(M >= 0 && K > 0 && ldf >= K && lds >= M, VITQ_ERR_INVALID_ARG);
  VITQ_CHECK(K % 16 == 0 && ldf % 8 == 0 && M <= VITQ_MAX_ROWS && K <= VITQ_MAX_DIM, VITQ_ERR_SHAPE);
  VITQ_CHECK(al16(f) && al16(q), VITQ_ERR_ALIGN);
  int sms = 0;
  int r = current_device_ok(&sms);
  if (r) return r;
  VITQ_LAUNCH("gelu_quant", S(stream), 0, quant_bytes(M, K),
              launch_gelu_quant((const __nv_bfloat16*)f, M, K, ldf, q, s, lds, sms, S(stream)));
  return VITQ_OK;
}

int fp8_block_gemm(const uint8_t* A, const float* sA, int ldsA, const uint8_t* W, const float* sW,
                   const void* bias, const void* residual, void* C, int M, int N, int K, void* stream) {
  VITQ_CHECK(A && sA && W && sW && C, VITQ_ERR_INVALID_ARG);
  VITQ_CHECK(M >= 0 && N > 0 && K > 0 && ldsA >= M, VITQ_ERR_INVALID_ARG);
  VITQ_CHECK(K % 16 == 0 && N % 8 == 0, VITQ_ERR_SHAPE);
  VITQ_CHECK(M <= VITQ_MAX_ROWS && N <= VITQ_MAX_DIM && K <= VITQ_MAX_DIM, VITQ_ERR_SHAPE);
  VITQ_CHECK(al16(A) && al16(W) && al16(C) && (!bias || al16(bias)) && (!residual || al16(residual)),
             VITQ_ERR_ALIGN);
  int sms = 0;
  int r = current_device_ok(&sms);
  if (r) return r;
  return gemm_checked(A, sA, ldsA, W, sW, bias, residual, C, M, N, K, sms, S(stream));
}

int bf16_gemm(const void* A, const void* W, const void* bias, const void* residual, void* C, int M, int N, int K,
              void* stream) {
  VITQ_CHECK(A && W && C, VITQ_ERR_INVALID_ARG);
  VITQ_CHECK(M >= 0 && N > 0 && K > 0, VITQ_ERR_INVALID_ARG);
  VITQ_CHECK(K % 8 == 0 && N % 8 == 0, VITQ_ERR_SHAPE);
  VITQ_CHECK(M <= VITQ_MAX_ROWS && N <= VITQ_MAX_DIM && K <= VITQ_MAX_DIM, VITQ_ERR_SHAPE);
  VITQ_CHECK(al16(A) && al16(W) && al16(C) && (!bias || al16(bias)) && (!residual || al16(residual)),
             VITQ_ERR_ALIGN);
  int sms = 0;
  int r = current_device_ok(&sms);
  if (r) return r;
  return bf16_gemm_checked((const __nv_bfloat16*)A, (const __nv_bfloat16*)W, (const __nv_bfloat16*)bias,
                           (const __nv_bfloat16*)residual, (__nv_bfloat16*)C, M, N, K, sms, S(stream));
}

int vit_rope_table(const int32_t* pos_hw, int n_tokens, float theta, float* cos_sin, void* stream) {
  VITQ_CHECK(pos_hw && cos_sin && n_tokens >= 0 && theta > 0.f, VITQ_ERR_INVALID_ARG);
  VITQ_CHECK(n_tokens <= VITQ_MAX_ROWS, VITQ_ERR_SHAPE);
  int r = current_device_ok(nullptr);
  if (r) return r;
  VITQ_LAUNCH("rope_table", S(stream), 0, (double)n_tokens * (8 + 288), launch_rope_table(pos_hw, n_tokens, (double)theta, cos_sin, S(stream)));
  return VITQ_OK;
}

int vit_rope2d(void* qkv, int n_tokens, const float* cos_sin, int flags, void* stream) {
  VITQ_CHECK(qkv && cos_sin && n_tokens >= 0 && (flags & ~VITQ_V_FP16) == 0, VITQ_ERR_INVALID_ARG);
  VITQ_CHECK(n_tokens <= VITQ_MAX_ROWS, VITQ_ERR_SHAPE);
  VITQ_CHECK(al16(qkv), VITQ_ERR_ALIGN);
  int r = current_device_ok(nullptr);
  if (r) return r;
  VITQ_LAUNCH("rope2d", S(stream), 0, (double)n_tokens * (2304 * 4 + 288), launch_rope_apply((__nv_bfloat16*)qkv, n_tokens, cos_sin, flags & VITQ_V_FP16, S(stream)));
  return VITQ_OK;
}

static int fill_grids(const int32_t* grid_hw, int n_images, bool need_even, GridList* g, int* n_total,
                      int* max_len) {
  VITQ_CHECK(grid_hw && n_images > 0 && n_images <= kMaxImages, VITQ_ERR_INVALID_ARG);
  g->n = n_images;
  long long tot = 0;
  int mx = 0;
  for (int i = 0; i < n_images; ++i) {
    const int h = grid_hw[2 * i], w = grid_hw[2 * i + 1];
    VITQ_CHECK(h > 0 && w > 0, VITQ_ERR_INVALID_ARG);
    if (need_even) VITQ_CHECK(h % 2 == 0 && w % 2 == 0, VITQ_ERR_SHAPE);
    const long long hw = (long long)h * w;   // 64-bit: h * w can exceed the int range
    VITQ_CHECK(hw <= VITQ_MAX_ROWS, VITQ_ERR_SHAPE);
    g->hw[2 * i] = h;
    g->hw[2 * i + 1] = w;
    tot += hw;
    VITQ_CHECK(tot <= VITQ_MAX_ROWS, VITQ_ERR_SHAPE);
    if (hw > mx) mx = (int)hw;
  }
  *n_total = (int)tot;
  *max_len = mx;
  return VITQ_OK;
}

int vit_positions(const int32_t* grid_hw, int n_images, int32_t* pos_hw, int32_t* cu_seqlens, void* stream) {
  VITQ_CHECK(pos_hw && cu_seqlens, VITQ_ERR_INVALID_ARG);
  GridList g;
  int n = 0, mx = 0;
  int r = fill_grids(grid_hw, n_images, false, &g, &n, &mx);
  if (r) return r;
  r = current_device_ok(nullptr);
  if (r) return r;
  VITQ_LAUNCH("positions", S(stream), 0, (double)n * 8, launch_positions(g, n, pos_hw, cu_seqlens, S(stream)));
  return VITQ_OK;
}

int vit_attention_varlen(const void* qkv, int n_tokens, const int32_t* cu_seqlens, int n_seqs, int max_seqlen,
                         float softmax_scale, int flags, void* out, void* stream) {
  VITQ_CHECK(qkv && cu_seqlens && out && (flags & ~VITQ_V_FP16) == 0, VITQ_ERR_INVALID_ARG);
  VITQ_CHECK(n_tokens >= 0 && n_seqs >= 0 && max_seqlen >= 0 && softmax_scale > 0.f, VITQ_ERR_INVALID_ARG);
  VITQ_CHECK(n_seqs <= 65535 && n_tokens <= VITQ_MAX_ROWS && max_seqlen <= VITQ_MAX_ROWS, VITQ_ERR_SHAPE);
  VITQ_CHECK(al16(qkv) && al16(out), VITQ_ERR_ALIGN);
  int r = current_device_ok(nullptr);
  if (r) return r;
  VITQ_LAUNCH("attention", S(stream), 0, (double)n_tokens * (3456 + 1152) * 2, launch_attention((const __nv_bfloat16*)qkv, n_tokens, cu_seqlens, n_seqs, max_seqlen, softmax_scale,
                            (flags & VITQ_V_FP16) != 0, (__nv_bfloat16*)out, S(stream)));
  return VITQ_OK;
}

size_t vitq_block_workspace_bytes(int n_tokens) {
  if (n_tokens < 0 || n_tokens > VITQ_MAX_ROWS) return 0;
  Carver c{nullptr};
  carve_block(c, n_tokens);
  return c.used;
}

size_t vitq_merger_workspace_bytes(int n_tokens) {
  if (n_tokens < 0 || n_tokens > VITQ_MAX_ROWS) return 0;
  Carver c{nullptr};
  carve_merger(c, n_tokens);
  return c.used;
}

size_t vitq_tower_workspace_bytes(int n_tokens_max, int n_images_max) {
  if (n_tokens_max < 0 || n_tokens_max > VITQ_MAX_ROWS || n_images_max < 1) return 0;
  Carver c{nullptr};
  carve_tower_head(c, n_tokens_max, n_images_max);
  Carver b{nullptr};
  carve_block(b, n_tokens_max);
  Carver m{nullptr};
  carve_merger(m, n_tokens_max);
  Carver mb{nullptr};
  carve_merger_bf16(mb, n_tokens_max);
  size_t scratch = b.used > m.used ? b.used : m.used;
  if (mb.used > scratch) scratch = mb.used;
  return c.used + scratch;
}

int vit_block_forward(const vitq_block_weights* w, void* x, int n_tokens, const int32_t* cu_seqlens, int n_seqs,
                      int max_seqlen, const float* cos_sin, void* ws, size_t ws_bytes, void* stream) {
  VITQ_CHECK(block_weights_ok(w), w ? VITQ_ERR_ALIGN : VITQ_ERR_INVALID_ARG);
  VITQ_CHECK(x && cu_seqlens && cos_sin && ws, VITQ_ERR_INVALID_ARG);
  VITQ_CHECK(n_tokens >= 0 && n_seqs >= 0 && max_seqlen >= 0, VITQ_ERR_INVALID_ARG);
  VITQ_CHECK(n_tokens <= VITQ_MAX_ROWS && max_seqlen <= VITQ_MAX_ROWS, VITQ_ERR_SHAPE);
  VITQ_CHECK(al16(x) && al16(ws), VITQ_ERR_ALIGN);
  VITQ_CHECK(ws_bytes >= vitq_block_workspace_bytes(n_tokens), VITQ_ERR_WORKSPACE);
  int sms = 0;
  int r = current_device_ok(&sms);
  if (r) return r;
  if (n_tokens == 0) return VITQ_OK;
  Carver c{reinterpret_cast<uint8_t*>(ws)};
  BlockWs b = carve_block(c, n_tokens);
  return block_impl(w, (__nv_bfloat16*)x, n_tokens, cu_seqlens, n_seqs, max_seqlen, cos_sin, b, sms, 0.0, S(stream));
}

int vit_merger_forward(const vitq_merger_weights* w, const void* x, int n_tokens, void* out, void* ws,
                       size_t ws_bytes, void* stream) {
  VITQ_CHECK(merger_weights_ok(w), w ? VITQ_ERR_ALIGN : VITQ_ERR_INVALID_ARG);
  VITQ_CHECK(x && out && ws && n_tokens >= 0, VITQ_ERR_INVALID_ARG);
  VITQ_CHECK(n_tokens % 4 == 0 && n_tokens <= VITQ_MAX_ROWS, VITQ_ERR_SHAPE);
  VITQ_CHECK(al16(x) && al16(out) && al16(ws), VITQ_ERR_ALIGN);
  VITQ_CHECK(ws_bytes >= vitq_merger_workspace_bytes(n_tokens), VITQ_ERR_WORKSPACE);
  int sms = 0;
  int r = current_device_ok(&sms);
  if (r) return r;
  if (n_tokens == 0) return VITQ_OK;
  Carver c{reinterpret_cast<uint8_t*>(ws)};
  MergerWs m = carve_merger(c, n_tokens);
  return merger_impl(w, (const __nv_bfloat16*)x, n_tokens, (__nv_bfloat16*)out, m, sms, S(stream));
}

}  // extern "C"

namespace vitq {
namespace {

// Tower driver ("Qwen3-VL-8B on RTX 5090", section 3, DeepStack taps; vision_encoder.rs,
// VisionEncoder): positions and rope table, then the 27 blocks with the 4 mergers
// after blocks 8, 16, 24 and 27.  run_block(blk, ...) and run_merger(tap, ...)
// pick each block's and merger's precision.
template <class BlockFn, class MergerFn>
int tower_drive(void* x, const int32_t* grid_hw, int n_images, void* const* taps, void* ws, size_t ws_bytes,
                void* stream, BlockFn run_block, MergerFn run_merger) {
  GridList g;
  int n = 0, max_len = 0;
  int r = fill_grids(grid_hw, n_images, true, &g, &n, &max_len);
  if (r) return r;
  VITQ_CHECK(al16(x) && al16(ws), VITQ_ERR_ALIGN);
  VITQ_CHECK(ws_bytes >= vitq_tower_workspace_bytes(n, n_images), VITQ_ERR_WORKSPACE);
  int sms = 0;
  r = current_device_ok(&sms);
  if (r) return r;
  cudaStream_t st = S(stream);
  Carver c{reinterpret_cast<uint8_t*>(ws)};
  TowerWs t = carve_tower_head(c, n, n_images);
  Carver rest{reinterpret_cast<uint8_t*>(ws) + c.used};
  BlockWs b = carve_block(rest, n);
  uint8_t* merger_ws = reinterpret_cast<uint8_t*>(ws) + c.used;   // aliases the block scratch
  VITQ_LAUNCH("positions", st, 0, (double)n * 8, launch_positions(g, n, t.pos, t.cu, st));
  VITQ_LAUNCH("rope_table", st, 0, (double)n * (8 + 288), launch_rope_table(t.pos, n, 10000.0, t.cs, st));
  double sumsq = 0;
  for (int i = 0; i < n_images; ++i) sumsq += (double)g.hw[2 * i] * g.hw[2 * i + 1] * g.hw[2 * i] * g.hw[2 * i + 1];
  static const int kTap[4] = {8, 16, 24, 27};
  int tap = 0;
  __nv_bfloat16* h = (__nv_bfloat16*)x;
  for (int blk = 1; blk <= VITQ_BLOCKS; ++blk) {
    r = run_block(blk, h, n, t.cu, n_images, max_len, t.cs, b, sms, sumsq, st);
    if (r) return r;
    if (tap < 4 && blk == kTap[tap]) {
      r = run_merger(tap, h, n, (__nv_bfloat16*)taps[tap], merger_ws, sms, st);
      if (r) return r;
      ++tap;
    }
  }
  return VITQ_OK;
}

}  // namespace
}  // namespace vitq

extern "C" {

int vit_tower_forward(const vitq_tower_weights* w, void* x, const int32_t* grid_hw, int n_images,
                      void* const* taps, void* ws, size_t ws_bytes, void* stream) {
  VITQ_CHECK(w && x && taps && ws, VITQ_ERR_INVALID_ARG);
  for (int t = 0; t < 4; ++t) VITQ_CHECK(taps[t] && al16(taps[t]), taps[t] ? VITQ_ERR_ALIGN : VITQ_ERR_INVALID_ARG);
  for (int b = 0; b < VITQ_BLOCKS; ++b)
    VITQ_CHECK(block_weights_ok(&w->blocks[b]), VITQ_ERR_INVALID_ARG);
  for (int t = 0; t < 4; ++t) VITQ_CHECK(merger_weights_ok(&w->mergers[t]), VITQ_ERR_INVALID_ARG);
  return tower_drive(
      x, grid_hw, n_images, taps, ws, ws_bytes, stream,
      [&](int blk, __nv_bfloat16* h, int n, const int32_t* cu, int ni, int ml, const float* cs, const BlockWs& b,
          int sms, double sumsq, cudaStream_t st) {
        return block_impl(&w->blocks[blk - 1], h, n, cu, ni, ml, cs, b, sms, sumsq, st);
      },
      [&](int tap, const __nv_bfloat16* h, int n, __nv_bfloat16* out, uint8_t* mws, int sms, cudaStream_t st) {
        Carver c{mws};
        return merger_impl(&w->mergers[tap], h, n, out, carve_merger(c, n), sms, st);
      });
}

int vit_tower_forward_mixed(const vitq_tower_weights_mixed* w, void* x, const int32_t* grid_hw, int n_images,
                            void* const* taps, void* ws, size_t ws_bytes, void* stream) {
  VITQ_CHECK(w && x && taps && ws, VITQ_ERR_INVALID_ARG);
  for (int t = 0; t < 4; ++t) VITQ_CHECK(taps[t] && al16(taps[t]), taps[t] ? VITQ_ERR_ALIGN : VITQ_ERR_INVALID_ARG);
  for (int b = 0; b < VITQ_BF16_HEAD_BLOCKS; ++b) VITQ_CHECK(block_bf16_weights_ok(&w->head[b]), VITQ_ERR_INVALID_ARG);
  for (int b = 0; b < VITQ_BLOCKS - VITQ_BF16_HEAD_BLOCKS; ++b)
    VITQ_CHECK(block_weights_ok(&w->blocks[b]), VITQ_ERR_INVALID_ARG);
  for (int t = 0; t < 4; ++t) VITQ_CHECK(merger_bf16_weights_ok(&w->mergers[t]), VITQ_ERR_INVALID_ARG);
  return tower_drive(
      x, grid_hw, n_images, taps, ws, ws_bytes, stream,
      [&](int blk, __nv_bfloat16* h, int n, const int32_t* cu, int ni, int ml, const float* cs, const BlockWs& b,
          int sms, double sumsq, cudaStream_t st) {
        if (blk <= VITQ_BF16_HEAD_BLOCKS)
          return block_bf16_impl(&w->head[blk - 1], h, n, cu, ni, ml, cs, b, sms, sumsq, st);
        return block_impl(&w->blocks[blk - 1 - VITQ_BF16_HEAD_BLOCKS], h, n, cu, ni, ml, cs, b, sms, sumsq, st);
      },
      [&](int tap, const __nv_bfloat16* h, int n, __nv_bfloat16* out, uint8_t* mws, int sms, cudaStream_t st) {
        Carver c{mws};
        return merger_bf16_impl(&w->mergers[tap], h, n, out, carve_merger_bf16(c, n), sms, st);
      });
}

int vit_block_forward_bf16(const vitq_block_weights_bf16* w, void* x, int n_tokens, const int32_t* cu_seqlens,
                           int n_seqs, int max_seqlen, const float* cos_sin, void* ws, size_t ws_bytes,
                           void* stream) {
  VITQ_CHECK(block_bf16_weights_ok(w), w ? VITQ_ERR_ALIGN : VITQ_ERR_INVALID_ARG);
  VITQ_CHECK(x && cu_seqlens && cos_sin && ws, VITQ_ERR_INVALID_ARG);
  VITQ_CHECK(n_tokens >= 0 && n_seqs >= 0 && max_seqlen >= 0, VITQ_ERR_INVALID_ARG);
  VITQ_CHECK(n_tokens <= VITQ_MAX_ROWS && max_seqlen <= VITQ_MAX_ROWS, VITQ_ERR_SHAPE);
  VITQ_CHECK(al16(x) && al16(ws), VITQ_ERR_ALIGN);
  VITQ_CHECK(ws_bytes >= vitq_block_workspace_bytes(n_tokens), VITQ_ERR_WORKSPACE);
  int sms = 0;
  int r = current_device_ok(&sms);
  if (r) return r;
  if (n_tokens == 0) return VITQ_OK;
  Carver c{reinterpret_cast<uint8_t*>(ws)};
  BlockWs b = carve_block(c, n_tokens);
  return block_bf16_impl(w, (__nv_bfloat16*)x, n_tokens, cu_seqlens, n_seqs, max_seqlen, cos_sin, b, sms, 0.0,
                         S(stream));
}

size_t vitq_patch_embed_workspace_bytes(int n_tokens) {
  if (n_tokens < 0 || n_tokens > VITQ_MAX_ROWS) return 0;
  return up256((size_t)n_tokens * VITQ_HIDDEN * 2);
}

int vit_patch_embed(const void* pixels, int n_tokens, const int32_t* grid_hw, int n_images, const void* w,
                    const void* b, const void* pos_table, void* x, void* ws, size_t ws_bytes, void* stream) {
  VITQ_CHECK(pixels && w && b && pos_table && x && ws && n_tokens >= 0, VITQ_ERR_INVALID_ARG);
  GridList g;
  int n = 0, max_len = 0;
  int r = fill_grids(grid_hw, n_images, false, &g, &n, &max_len);
  if (r) return r;
  VITQ_CHECK(n == n_tokens, VITQ_ERR_SHAPE);
  VITQ_CHECK(al16(pixels) && al16(w) && al16(b) && al16(pos_table) && al16(x) && al16(ws), VITQ_ERR_ALIGN);
  VITQ_CHECK(ws_bytes >= vitq_patch_embed_workspace_bytes(n_tokens), VITQ_ERR_WORKSPACE);
  int sms = 0;
  r = current_device_ok(&sms);
  if (r) return r;
  if (n_tokens == 0) return VITQ_OK;
  cudaStream_t st = S(stream);
  __nv_bfloat16* pos = reinterpret_cast<__nv_bfloat16*>(ws);
  VITQ_LAUNCH("pos_interp", st, 0, (double)n_tokens * VITQ_HIDDEN * (4 * 2 + 2),
              launch_pos_interp(g, n_tokens, (const __nv_bfloat16*)pos_table, pos, st));
  return bf16_gemm_checked((const __nv_bfloat16*)pixels, (const __nv_bfloat16*)w, (const __nv_bfloat16*)b, pos,
                           (__nv_bfloat16*)x, n_tokens, VITQ_HIDDEN, VITQ_PATCH_DIM, sms, st);
}

size_t vitq_merger_bf16_workspace_bytes(int n_tokens) {
  if (n_tokens < 0 || n_tokens > VITQ_MAX_ROWS) return 0;
  Carver c{nullptr};
  carve_merger_bf16(c, n_tokens);
  return c.used;
}

int vit_merger_forward_bf16(const vitq_merger_weights_bf16* w, const void* x, int n_tokens, void* out, void* ws,
                            size_t ws_bytes, void* stream) {
  VITQ_CHECK(merger_bf16_weights_ok(w), w ? VITQ_ERR_ALIGN : VITQ_ERR_INVALID_ARG);
  VITQ_CHECK(x && out && ws && n_tokens >= 0, VITQ_ERR_INVALID_ARG);
  VITQ_CHECK(n_tokens % 4 == 0 && n_tokens <= VITQ_MAX_ROWS, VITQ_ERR_SHAPE);
  VITQ_CHECK(al16(x) && al16(out) && al16(ws), VITQ_ERR_ALIGN);
  VITQ_CHECK(ws_bytes >= vitq_merger_bf16_workspace_bytes(n_tokens), VITQ_ERR_WORKSPACE);
  int sms = 0;
  int r = current_device_ok(&sms);
  if (r) return r;
  if (n_tokens == 0) return VITQ_OK;
  Carver c{reinterpret_cast<uint8_t*>(ws)};
  MergerBf16Ws m = carve_merger_bf16(c, n_tokens);
  return merger_bf16_impl(w, (const __nv_bfloat16*)x, n_tokens, (__nv_bfloat16*)out, m, sms, S(stream));
}

int vitq_get_device_error(void* stream) {
  if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return VITQ_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)) != cudaSuccess) return VITQ_ERR_CUDA;
  const unsigned int zero = 0;
  if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess) return VITQ_ERR_CUDA;
  if (v & kErrWaitTimeout) return VITQ_ERR_DEVICE_TIMEOUT;
  return v ? VITQ_ERR_RANGE : VITQ_OK;
}

const char* vitq_status_string(int s) {
  switch (s) {
    case VITQ_OK: return "ok";
    case VITQ_ERR_INVALID_ARG: return "invalid argument";
    case VITQ_ERR_SHAPE: return "unsupported shape";
    case VITQ_ERR_ALIGN: return "pointer not 16-byte aligned";
    case VITQ_ERR_ARCH: return "device is not sm_100";
    case VITQ_ERR_CUDA: return "CUDA error";
    case VITQ_ERR_WORKSPACE: return "workspace too small";
    case VITQ_ERR_DEVICE_TIMEOUT: return "device pipeline wait timed out";
    case VITQ_ERR_RANGE: return "value beyond the range of its format (clamped)";
    default: return "unknown status";
  }
}

unsigned long long vitq_launch_count(void) { return g_launches.load(); }

#ifdef VITQ_TRACE
// Development builds only: copies the [32][4096] clock table (0 = no event) and clears it.
int vitq_trace_read(unsigned long long* out, int cap) {
  cudaDeviceSynchronize();
  const int n = (int)(kTraceTags * kTracePerTag);
  if (cap < n) return -1;
  cudaMemcpyFromSymbol(out, g_trace, (size_t)n * 8);
  static std::vector<unsigned long long> zero((size_t)n, 0ull);
  cudaMemcpyToSymbol(g_trace, zero.data(), (size_t)n * 8);
  return n;
}
#endif

void vitq_profile_start(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto& r : g_prof) {
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  g_prof.clear();
  g_prof_ms.clear();
  g_prof_on = true;
}

int vitq_profile_stop(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_on = false;
  g_prof_ms.assign(g_prof.size(), 0.f);
  for (size_t i = 0; i < g_prof.size(); ++i) {
    // negative on failure, so that an error is never read as a record count
    if (cudaEventSynchronize(g_prof[i].b) != cudaSuccess) return -VITQ_ERR_CUDA;
    if (cudaEventElapsedTime(&g_prof_ms[i], g_prof[i].a, g_prof[i].b) != cudaSuccess) return -VITQ_ERR_CUDA;
  }
  return (int)g_prof.size();
}

int vitq_profile_get(int i, const char** name, float* ms, double* flops, double* bytes) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (i < 0 || (size_t)i >= g_prof_ms.size() || !name || !ms || !flops || !bytes) return VITQ_ERR_INVALID_ARG;
  *name = g_prof[i].name;
  *ms = g_prof_ms[i];
  *flops = g_prof[i].flops;
  *bytes = g_prof[i].bytes;
  return VITQ_OK;
}

int vitq_selftest_wait_timeout(int limit_us, void* stream) {
  VITQ_CHECK(limit_us > 0 && limit_us <= 1000000, VITQ_ERR_INVALID_ARG);
  int r = current_device_ok(nullptr);
  if (r) return r;
  VITQ_LAUNCH("selftest_wait", S(stream), 0, 0, launch_selftest_wait(limit_us, S(stream)));
  return VITQ_OK;
}

}  // extern "C"
