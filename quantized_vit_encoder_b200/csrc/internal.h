// Internal launchers shared by the C-ABI layer (not part of the public ABI).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdlib>
#include <utility>

namespace vitq {

// Launch on `st` with programmatic stream serialisation (the kernel overlaps its
// scheduling with the previous kernel's tail and waits for it with pdl_wait).
// VITQ_PDL=0 in the environment launches without it.
inline bool pdl_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("VITQ_PDL");
    return !(e && e[0] == '0');
  }();
  return on;
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}


constexpr int kMaxImages = 64;

// Patch grids passed by value to the positions kernel.
struct GridList {
  int n;
  int hw[2 * kMaxImages];
};

// TMA tensor-map encoders (host).
// 2D uint8 matrix [rows, cols] (row pitch = cols bytes), box {box_cols, box_rows}, 128B swizzle.
cudaError_t encode_tma_2d_u8(CUtensorMap* tm, const void* base, int cols, int rows, int box_cols,
                             int box_rows);
// 2D bf16 matrix [rows, cols] (row pitch = cols * 2 bytes), box {box_cols, box_rows}, 128B swizzle
// (box_cols = 64).
cudaError_t encode_tma_2d_bf16(CUtensorMap* tm, const void* base, int cols, int rows, int box_cols,
                               int box_rows);
// Packed qkv [n, 3, 16, 72] bf16 viewed as 3D (d = 72, slot = 48, token = n); box {box_d, 1, 128}.
// lo = true: 128B swizzle (box_d = 64); lo = false: 32B swizzle (box_d = 16).
cudaError_t encode_tma_qkv(CUtensorMap* tm, const void* qkv, int n_tokens, int box_d, bool lo);

cudaError_t launch_quant_act(const __nv_bfloat16* x, int M, int K, int ldx, uint8_t* q, float* s,
                             int lds, cudaStream_t st);
cudaError_t launch_ln_quant(const __nv_bfloat16* x, int ldx, const __nv_bfloat16* gamma,
                            const __nv_bfloat16* beta, int M, int K, double eps, uint8_t* q,
                            float* s, int lds, cudaStream_t st);
// LayerNorm / GELU with either FP8 output (q, s) or bf16 output (y, when not null).
cudaError_t launch_ln(const __nv_bfloat16* x, int ldx, const __nv_bfloat16* gamma, const __nv_bfloat16* beta,
                      int M, int K, double eps, uint8_t* q, float* s, int lds, __nv_bfloat16* y,
                      cudaStream_t st);
cudaError_t launch_gelu(const __nv_bfloat16* f, int M, int K, int ldf, uint8_t* q, float* s, int lds,
                        __nv_bfloat16* y, int num_sms, cudaStream_t st);
// One-time per device: GELU of every bf16 value into the device table.
cudaError_t build_gelu_table(cudaStream_t st);
cudaError_t launch_gelu_quant(const __nv_bfloat16* f, int M, int K, int ldf, uint8_t* q, float* s,
                              int lds, int num_sms, cudaStream_t st);
cudaError_t launch_quant_weight(const __nv_bfloat16* w, int N, int K, uint8_t* q, float* s,
                                cudaStream_t st);
cudaError_t launch_rope_table(const int32_t* pos, int n, double theta, float* cs, cudaStream_t st);
cudaError_t launch_rope_apply(__nv_bfloat16* qkv, int n, const float* cs, int v_to_f16, cudaStream_t st);
// Bilinear interpolation of the 48 x 48 position table to each packed token's (row, col).
cudaError_t launch_pos_interp(const GridList& g, int n_total, const __nv_bfloat16* table, __nv_bfloat16* out,
                              cudaStream_t st);
cudaError_t launch_positions(const GridList& g, int n_total, int32_t* pos, int32_t* cu,
                             cudaStream_t st);
cudaError_t launch_fp8_gemm(const uint8_t* A, const float* sA, int ldsA, const uint8_t* W, const float* sW,
                            const __nv_bfloat16* bias, const __nv_bfloat16* residual, __nv_bfloat16* C,
                            int M, int N, int K, int block_n, bool pair, int num_sms, cudaStream_t st);
// bf16 GEMM: C = A W^T + bias + residual (fp32 accumulation), A [M, K], W [N, K].
cudaError_t launch_bf16_gemm(const __nv_bfloat16* A, const __nv_bfloat16* W, const __nv_bfloat16* bias,
                             const __nv_bfloat16* residual, __nv_bfloat16* C, int M, int N, int K, int block_n,
                             int num_sms, cudaStream_t st);
cudaError_t launch_attention(const __nv_bfloat16* qkv, int n_tokens, const int32_t* cu, int n_seqs,
                             int max_seqlen, float scale, bool v_f16, __nv_bfloat16* out, cudaStream_t st);

cudaError_t launch_selftest_wait(int limit_us, cudaStream_t st);

}  // namespace vitq
