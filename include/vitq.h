/*
 * vitq — FP8 ViT vision-tower forward pass for NVIDIA B200 (sm_100a).
 *
 * C ABI of libvitq.so.  Every computation runs in CUDA kernels of this library
 * on the caller's stream; there is no host fallback.
 *
 * Conventions for every entry point
 * ---------------------------------
 *  - Pointers are DEVICE pointers unless a parameter says "host".  The caller
 *    owns all memory; the library never allocates, frees or synchronises the
 *    host (except vitq_get_device_error, which reads a device word, and the
 *    one-time setup below).
 *  - The first call on each device that reaches the device checks its
 *    architecture and fills the library's GELU table on that device (a 128 KB
 *    array of the library, one kernel on a private stream, waited for).  Make
 *    that first call before any stream capture begins.  This per-device state
 *    (and the scratch address of vit_merger_forward_static) is kept for the
 *    life of the process and assumes the device's primary context lives as
 *    long: after cudaDeviceReset the library's device arrays are gone, so
 *    the library must not be called again in that process.
 *  - bf16 tensors are passed as `const void*` / `void*` holding IEEE bfloat16
 *    values; FP8 codes are OCP E4M3 ("E4M3FN") bytes; scales are fp32.
 *  - Matrices are row-major.  Activation FP8 codes are [M, K] (K contiguous);
 *    activation scales are kb-major: s[kb * lds + m] for K block kb = k / 128
 *    (one scale per row per 128 columns, the last block may be shorter).
 *    Weight codes are [N, K]; weight scales are [ceil(N/128), ceil(K/128)].
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).
 *  - Arguments are validated on the host before anything is launched; on an
 *    error nothing is launched and a vitq_status below is returned.
 *  - Pointers passed to the GEMM / attention paths must be 16-byte aligned.
 *  - Kernels are launched with programmatic dependent launch: each may start
 *    while the previous kernel on the stream finishes, and waits for it before
 *    reading its inputs.  Two reads happen before that wait: LayerNorm's gamma
 *    and beta (vit_ln_quant, vit_block_forward, the mergers) and attention's
 *    cu_seqlens (vit_attention_varlen).  So these must not be written by the
 *    kernel launched immediately before the call on the same stream (weights
 *    and segment offsets normally are not); otherwise put any stream-ordered
 *    operation between, or set VITQ_PDL=0 in the environment.
 *
 * Sources (web pages; the section named is where each step is described):
 *  [FRT] "Qwen3-VL-8B on RTX 5090 (NVFP4 language stack + FP8 ViT)"
 *  [VE]  "spark_model/layers/vision_encoder.rs" (struct definitions)
 *  [TRT] "qwen3_omni: record why FP8 is not shipped" (FP8 scale amax / 448)
 */
#ifndef VITQ_H_
#define VITQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  VITQ_OK = 0,
  VITQ_ERR_INVALID_ARG = 1,   /* null pointer, negative count, bad flag */
  VITQ_ERR_SHAPE = 2,         /* unsupported dimension (K % 16, odd grid for the merger, ...) */
  VITQ_ERR_ALIGN = 3,         /* pointer not 16-byte aligned */
  VITQ_ERR_ARCH = 4,          /* current device is not sm_100 */
  VITQ_ERR_CUDA = 5,          /* a CUDA call or kernel launch failed */
  VITQ_ERR_WORKSPACE = 6,     /* workspace smaller than the *_workspace_bytes figure */
  VITQ_ERR_DEVICE_TIMEOUT = 7, /* a kernel's bounded pipeline wait expired (see vitq_get_device_error) */
  VITQ_ERR_RANGE = 8           /* a value beyond its storage format was clamped (see vitq_get_device_error) */
} vitq_status;

/* Model dimensions (Qwen3-VL vision tower: [FRT] section 3, [VE] VisionEncoder). */
#define VITQ_HIDDEN 1152
#define VITQ_HEADS 16
#define VITQ_HEAD_DIM 72
#define VITQ_MLP 4304
#define VITQ_QKV 3456
#define VITQ_MERGE_IN 4608
#define VITQ_OUT_HIDDEN 2048
#define VITQ_BLOCKS 27
#define VITQ_MAX_IMAGES 64

/* Size limits, checked on the host by every entry point (VITQ_ERR_SHAPE beyond
 * them; the *_workspace_bytes functions return 0).  Within them every index the
 * kernels form in 32-bit arithmetic (rows x 36 rotary items, rows x 32 lanes,
 * tile counts, (M + 127) / 128) stays in the int range. */
#define VITQ_MAX_ROWS (1 << 24) /* M, n_tokens, max_seqlen, and a tower's total patch count */
#define VITQ_MAX_DIM (1 << 16)  /* N and K of the GEMM and quantisation primitives */

/* Weights of one ViT block ([VE] ViTBlock): LayerNorm gamma/beta and biases are
 * bf16; each linear is FP8 codes [out, in] plus fp32 128x128 block scales. */
typedef struct {
  const void* norm1_w; const void* norm1_b;                   /* [1152] */
  const uint8_t* qkv_q; const float* qkv_s; const void* qkv_b;  /* [3456,1152], [27,9], [3456] */
  const uint8_t* proj_q; const float* proj_s; const void* proj_b; /* [1152,1152], [9,9], [1152] */
  const void* norm2_w; const void* norm2_b;                   /* [1152] */
  const uint8_t* fc1_q; const float* fc1_s; const void* fc1_b;  /* [4304,1152], [34,9], [4304] */
  const uint8_t* fc2_q; const float* fc2_s; const void* fc2_b;  /* [1152,4304], [9,34], [1152] */
} vitq_block_weights;

/* Weights of one 2x2 patch merger ([VE] MergerLayer). */
typedef struct {
  const void* norm_w; const void* norm_b;                     /* [4608] */
  const uint8_t* fc1_q; const float* fc1_s; const void* fc1_b;  /* [4608,4608], [36,36], [4608] */
  const uint8_t* fc2_q; const float* fc2_s; const void* fc2_b;  /* [2048,4608], [16,36], [2048] */
} vitq_merger_weights;

/* Whole tower ([VE] VisionEncoder): 27 blocks and 4 mergers (after blocks 8, 16, 24, 27). */
typedef struct {
  vitq_block_weights blocks[VITQ_BLOCKS];
  vitq_merger_weights mergers[4];
} vitq_tower_weights;

/* bf16 variants ([FRT] s4: a massive-activation channel makes the image
 * embeddings sensitive to FP8, so the first three blocks and the mergers keep
 * bf16 weights and activations).  Same layout as above with bf16 weight
 * matrices [out, in] instead of FP8 codes and scales. */
typedef struct {
  const void* norm1_w; const void* norm1_b;  /* [1152] */
  const void* qkv_w; const void* qkv_b;      /* [3456,1152], [3456] */
  const void* proj_w; const void* proj_b;    /* [1152,1152], [1152] */
  const void* norm2_w; const void* norm2_b;  /* [1152] */
  const void* fc1_w; const void* fc1_b;      /* [4304,1152], [4304] */
  const void* fc2_w; const void* fc2_b;      /* [1152,4304], [1152] */
} vitq_block_weights_bf16;

typedef struct {
  const void* norm_w; const void* norm_b;    /* [4608] */
  const void* fc1_w; const void* fc1_b;      /* [4608,4608], [4608] */
  const void* fc2_w; const void* fc2_b;      /* [2048,4608], [2048] */
} vitq_merger_weights_bf16;

/* Mixed-precision tower: blocks 1-3 and the 4 mergers bf16, blocks 4-27 FP8. */
#define VITQ_BF16_HEAD_BLOCKS 3
typedef struct {
  vitq_block_weights_bf16 head[VITQ_BF16_HEAD_BLOCKS];
  vitq_block_weights blocks[VITQ_BLOCKS - VITQ_BF16_HEAD_BLOCKS];
  vitq_merger_weights_bf16 mergers[4];
} vitq_tower_weights_mixed;

/* ---------------------------------------------------------------- stages */

/* 1x128 FP8 activation quantisation ([FRT] s3: activations quantised per token
 * and per 128-column K block; scale convention [TRT]).  x: bf16 [M, ldx] (first K
 * columns used).  For each row m and K block kb: s = amax / 448 (fp32 IEEE
 * division), q = E4M3_RNE_satfinite(x / s); a zero scale gives zero codes.
 * Outputs q [M, K] and s[kb * lds + m].  K % 16 == 0, lds >= M. */
int vit_quant_act(const void* x, int M, int K, int ldx, uint8_t* q, float* s, int lds, void* stream);

/* 128x128-block FP8 weight quantisation ([FRT] introduction: block-128 W8A8
 * linears; scale convention [TRT]) (same convention, one scale per block).
 * w: bf16 [N, K] -> q [N, K], s [ceil(N/128), ceil(K/128)].  Set-up step. */
int vit_quant_weight(const void* w, int N, int K, uint8_t* q, float* s, void* stream);

/* LayerNorm (biased variance, eps) with the bf16 result quantised as in
 * vit_quant_act ([FRT] s3 layer_norm_to_fp8_block128: the bf16 normalised
 * activation never goes to HBM).  Statistics and the affine step in fp64,
 * one rounding to bf16.  x: bf16 [M, ldx]; gamma/beta bf16 [K]; K <= 4608. */
int vit_ln_quant(const void* x, int M, int K, int ldx, const void* gamma, const void* beta, float eps,
                 uint8_t* q, float* s, int lds, void* stream);

/* GELU(tanh) of a bf16 activation, rounded to bf16, quantised as in
 * vit_quant_act ([FRT] s3 gelu_tanh_to_fp8_block128).  f: bf16 [M, ldf].
 * The bf16 GELU of each input is read from a table holding, for every bf16
 * value, the bf16 rounding of the fp64 value x / (1 + exp(-2u)). */
int vit_gelu_quant(const void* f, int M, int K, int ldf, uint8_t* q, float* s, int lds, void* stream);

/* FP8 W8A8 block-scaled GEMM with fused bias and residual ([FRT] s1: the ViT
 * linears run as FP8 block-128 GEMMs with the bias add fused; [VE] vision_gemm_bias):
 *   C[m,n] = bf16( sum_kb sA[kb*ldsA+m] * sW[(n/128)*ceil(K/128)+kb] * sum_{k in kb} A[m,k] W[n,k]
 *                  + bias[n] + residual[m,n] )
 * A: E4M3 [M, K]; W: E4M3 [N, K]; bias bf16 [N] or NULL; residual bf16 [M, N]
 * or NULL (may equal C); C bf16 [M, N].  K % 16 == 0, N % 8 == 0, ldsA >= M.
 * The K tail (K % 128) is zero-filled in shared memory, so K needs no padding. */
int fp8_block_gemm(const uint8_t* A, const float* sA, int ldsA, const uint8_t* W, const float* sW,
                   const void* bias, const void* residual, void* C, int M, int N, int K, void* stream);

/* bf16 GEMM with fused bias and residual, fp32 accumulation over all of K
 * ([FRT] s4: the patch embedding, the first three blocks and the mergers stay
 * bf16; [VE] dense_gemm_bf16 / vision_gemm_bias):
 *   C[m,n] = bf16( sum_k A[m,k] W[n,k] + bias[n] + residual[m,n] )
 * A: bf16 [M, K]; W: bf16 [N, K]; bias bf16 [N] or NULL; residual bf16 [M, N]
 * or NULL (may equal C); C bf16 [M, N].  K % 8 == 0, N % 8 == 0; all pointers
 * 16-byte aligned.  The K tail (K % 64) is zero-filled in shared memory. */
int bf16_gemm(const void* A, const void* W, const void* bias, const void* residual, void* C, int M, int N, int K,
              void* stream);

/* 2D rotary table ([FRT] s3: 2D rotary in rotate_half form; [VE] rope_inv_freq, head_dim/4
 * entries).  pos_hw: int32 [n][2] (row, col) per token.  Output cos_sin fp32
 * [n][72]: cos of the 36 angles then their sines; angle j = row * f_j for
 * j < 18 and col * f_(j-18) otherwise, f_i = theta^(-2i/36).  fp64 inside. */
int vit_rope_table(const int32_t* pos_hw, int n_tokens, float theta, float* cos_sin, void* stream);

/* Flag for vit_rope2d / vit_attention_varlen: the v part of qkv is (made) fp16.
 * v comes out of a bf16 GEMM; bf16 -> fp16 (round to nearest) is exact for
 * 2^-14 <= |v| < 65504 and off by at most 2^-25 below that, and the
 * attention then runs its P.V product with fp16 P (11 significant bits instead
 * of 8) at the same tensor-core rate. */
#define VITQ_V_FP16 1

/* 2D rotary ([FRT] s3, applied after the QKV projection; [VE] head_dim 72).
 * Apply the rotary in place to the q and k parts of qkv bf16 [n, 3, 16, 72]:
 * pairs (j, j+36): x'_j = x_j cos - x_(j+36) sin, x'_(j+36) = x_(j+36) cos + x_j sin,
 * fp32 arithmetic, one rounding to bf16.  flags = VITQ_V_FP16 also converts the
 * v part to fp16 in place; flags = 0 leaves it untouched. */
int vit_rope2d(void* qkv, int n_tokens, const float* cos_sin, int flags, void* stream);

/* Patch positions of packed images ([FRT] s5: one attention window per image).
 * grid_hw: HOST int32 [n_images][2] (h, w).  Writes pos_hw int32 [n][2] and
 * cu_seqlens int32 [n_images + 1].  Token order: 2x2-block order for even
 * grids (the merger's 4 neighbours are consecutive rows), row-major otherwise. */
int vit_positions(const int32_t* grid_hw, int n_images, int32_t* pos_hw, int32_t* cu_seqlens,
                  void* stream);

/* Block-diagonal non-causal attention ([FRT] s1/s3: full, bidirectional
 * flash attention per block; s5: cu_seqlens).  qkv: bf16 [n_tokens, 3, 16, 72] (rotary already applied);
 * cu_seqlens int32 [n_seqs + 1] with cu[0] = 0, cu[n_seqs] = n_tokens;
 * max_seqlen >= every segment length.  cu_seqlens lives in device memory and
 * is read only by the kernel, so the host cannot check it: it must be
 * non-decreasing from 0 (rows past n_tokens are neither read nor written;
 * query rows of a segment past max_seqlen are left unwritten).  out: bf16
 * [n_tokens, 1152], head h in
 * columns h*72 .. h*72+71.  qkv must be 16-byte aligned.  flags: 0 = v is bf16
 * and P is rounded to bf16 for P.V (flash-attention bf16 numerics);
 * VITQ_V_FP16 = v is fp16 (see vit_rope2d) and P is rounded to fp16. */
int vit_attention_varlen(const void* qkv, int n_tokens, const int32_t* cu_seqlens, int n_seqs,
                         int max_seqlen, float softmax_scale, int flags, void* out, void* stream);

/* Patch embedding with the interpolated position embedding ([FRT] s3: the
 * patch embedding is followed by the add of the interpolated position table; [VE] PATCH_DIM = 3*2*16*16 = 1536,
 * patch_embed_w [1152, 1536], pos_embed [2304, 1152], num_grid_per_side 48):
 *   x[t] = bf16( pixels[t] . w^T + b + pos[t] ),
 * pos[t] = bf16(bilinear interpolation of the 48 x 48 table at the token's
 * (row, col)), sample points running corner to corner (row r of an h-row grid
 * at table row r * 47 / (h - 1)).  pixels: bf16 [n_tokens, 1536], patchified,
 * in the tower's token order (see vit_positions); grid_hw: HOST int32
 * [n_images][2] with sum h*w == n_tokens (any h, w); w bf16 [1152, 1536];
 * b bf16 [1152]; pos_table bf16 [2304, 1152]; x bf16 [n_tokens, 1152] (output).
 * ws >= vitq_patch_embed_workspace_bytes(n_tokens).  All 16-byte aligned. */
int vit_patch_embed(const void* pixels, int n_tokens, const int32_t* grid_hw, int n_images, const void* w,
                    const void* b, const void* pos_table, void* x, void* ws, size_t ws_bytes, void* stream);
size_t vitq_patch_embed_workspace_bytes(int n_tokens);
#define VITQ_PATCH_DIM 1536
#define VITQ_POS_GRID 48

/* ---------------------------------------------------------------- layers */

/* One ViT block in place on x bf16 [n_tokens, 1152] ([FRT] s3 per-block chain):
 * LN1+quant -> QKV GEMM+bias -> RoPE -> attention -> quant -> proj GEMM+bias+x
 * -> LN2+quant -> fc1 GEMM+bias -> GELU+quant -> fc2 GEMM+bias+residual.
 * cu_seqlens, n_seqs, max_seqlen as for vit_attention_varlen (device memory,
 * not checked by the host); cos_sin from vit_rope_table, fp32 [n_tokens, 72];
 * ws >= vitq_block_workspace_bytes(n_tokens). */
int vit_block_forward(const vitq_block_weights* w, void* x, int n_tokens, const int32_t* cu_seqlens,
                      int n_seqs, int max_seqlen, const float* cos_sin, void* ws, size_t ws_bytes,
                      void* stream);
size_t vitq_block_workspace_bytes(int n_tokens);

/* 2x2 spatial merger ([FRT] s3: the 2x2 merger on each tap; [VE] MergerLayer): rows
 * 4i..4i+3 of x bf16 [n_tokens, 1152] form one 4608 row; LayerNorm(4608)+quant
 * -> fc1 4608->4608 + bias -> GELU+quant -> fc2 4608->2048 + bias.
 * out: bf16 [n_tokens/4, 2048].  n_tokens % 4 == 0.
 * ws >= vitq_merger_workspace_bytes(n_tokens). */
int vit_merger_forward(const vitq_merger_weights* w, const void* x, int n_tokens, void* out, void* ws,
                       size_t ws_bytes, void* stream);
size_t vitq_merger_workspace_bytes(int n_tokens);

/* The merger above with no workspace argument and no allocation of any kind.
 * This entry point has no counterpart in the sources: it serves callers that
 * may not allocate device memory, or pass a buffer, once running (code inside
 * an allocator callback, a plugin host that forbids allocations after
 * start-up, a serving loop that must never reach cudaMalloc, which can
 * synchronise the whole device).  Its scratch is one fixed array per device,
 * part of this library, sized for VITQ_MERGER_STATIC_MAX_TOKENS input tokens
 * (about 13.6 MiB).
 *  - n_tokens > VITQ_MERGER_STATIC_MAX_TOKENS returns VITQ_ERR_WORKSPACE and
 *    launches nothing; other arguments as vit_merger_forward.
 *  - The first call on each device, with that device current, looks up the
 *    array's device address (and may load this library's kernels there, and
 *    does the one-time setup described at the top of this file).  Make that
 *    first call before any stream capture begins.
 *  - All calls on one device share the array.  Calls issued in order on one
 *    stream are safe; calls that can overlap (different streams, or host
 *    threads, without ordering between them) race on it and corrupt each
 *    other's results.
 *  - Nothing in the array needs to start at zero. */
#define VITQ_MERGER_STATIC_MAX_TOKENS 4096
int vit_merger_forward_static(const vitq_merger_weights* w, const void* x, int n_tokens, void* out,
                              void* stream);

/* The 27-block tower over packed images with DeepStack taps ([FRT] s3: DeepStack
 * taps after layers 8, 16 and 24; [VE] deepstack_indexes [8,16,24] + final merger).
 * x: bf16 [n, 1152] patch embeddings, overwritten with the block-27 output.
 * grid_hw: HOST int32 [n_images][2], every h and w even.  taps[t]: bf16
 * [n/4, 2048] outputs of merger t (after blocks 8, 16, 24, 27).
 * ws >= vitq_tower_workspace_bytes(n, n_images). */
int vit_tower_forward(const vitq_tower_weights* w, void* x, const int32_t* grid_hw, int n_images,
                      void* const* taps, void* ws, size_t ws_bytes, void* stream);
size_t vitq_tower_workspace_bytes(int n_tokens_max, int n_images_max);

/* bf16 block ([FRT] s4: the first three blocks keep bf16 weights and
 * activations; the per-block chain of [FRT] s3), in place on x bf16
 * [n_tokens, 1152]: LN1 (bf16) -> QKV bf16 GEMM + bias -> RoPE -> attention ->
 * proj bf16 GEMM + bias + x -> LN2 (bf16) -> fc1 bf16 GEMM + bias -> GELU (bf16)
 * -> fc2 bf16 GEMM + bias + residual.  Arguments as vit_block_forward;
 * ws >= vitq_block_workspace_bytes(n_tokens). */
int vit_block_forward_bf16(const vitq_block_weights_bf16* w, void* x, int n_tokens, const int32_t* cu_seqlens,
                           int n_seqs, int max_seqlen, const float* cos_sin, void* ws, size_t ws_bytes,
                           void* stream);

/* bf16 2x2 merger ([FRT] s4: the mergers keep bf16): as vit_merger_forward
 * with bf16 LayerNorm output, bf16 fc1 and fc2 and a bf16 GELU.
 * ws >= vitq_merger_bf16_workspace_bytes(n_tokens). */
int vit_merger_forward_bf16(const vitq_merger_weights_bf16* w, const void* x, int n_tokens, void* out, void* ws,
                            size_t ws_bytes, void* stream);
size_t vitq_merger_bf16_workspace_bytes(int n_tokens);

/* The tower with blocks 1-3 and the mergers in bf16 ([FRT] s4).  Arguments as
 * vit_tower_forward; ws >= vitq_tower_workspace_bytes(n, n_images). */
int vit_tower_forward_mixed(const vitq_tower_weights_mixed* w, void* x, const int32_t* grid_hw, int n_images,
                            void* const* taps, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- status */

/* Reads and clears the device error word after synchronising `stream`:
 * 0 = none, VITQ_ERR_DEVICE_TIMEOUT = a bounded pipeline wait expired (reported
 * first when both happened), VITQ_ERR_RANGE = a v value beyond +-65504 was
 * clamped by the fp16 conversion (vit_rope2d with VITQ_V_FP16, the block
 * paths), VITQ_ERR_CUDA if synchronising the stream failed. */
int vitq_get_device_error(void* stream);
/* A static English description of a vitq_status ("unknown status" otherwise). */
const char* vitq_status_string(int status);
/* Number of kernel launches issued by this library since load (diagnostic). */
unsigned long long vitq_launch_count(void);

/* Launch timing.  Between vitq_profile_start and vitq_profile_stop every kernel
 * launch of this library is bracketed by a CUDA event pair on its stream (not
 * for use during stream capture).  vitq_profile_stop waits for the events and
 * returns the number of records (-VITQ_ERR_CUDA if an event cannot be read);
 * vitq_profile_get returns record i (VITQ_ERR_INVALID_ARG past the last): the kernel
 * name (static string), its device time in ms, and its algorithmic FLOPs and
 * HBM bytes (0 where the host does not know them). */
void vitq_profile_start(void);
int vitq_profile_stop(void);
int vitq_profile_get(int i, const char** name, float* ms, double* flops, double* bytes);

/* Runs a one-CTA kernel whose pipeline wait can never complete, with a limit of
 * limit_us microseconds (1..1e6): the wait gives up, sets the device error word
 * and the kernel returns, so vitq_get_device_error then reports
 * VITQ_ERR_DEVICE_TIMEOUT.  Checks the timeout path; hangs nothing. */
int vitq_selftest_wait_timeout(int limit_us, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* VITQ_H_ */
