// Block-diagonal non-causal attention over packed images, head_dim 72, on the
// sm_100a tensor cores.
//
// "Qwen3-VL-8B on RTX 5090", section 3 (FA2 full bidirectional attention per
// ViT block) and section 5 (each image is its own attention window, packed
// with cu_seqlens): O = softmax(Q K^T * scale) V per segment and head.
//
// Design (B200):
//   * one CTA per (segment, head, 128-query tile); 6 warps: TMA producer, MMA
//     issuer, 4 softmax warps (one thread per query row = one TMEM lane);
//   * Q, K, V are read straight from the packed qkv activation [n, 3, 16, 72]
//     through 3D TMA maps (d, slot, token).  head_dim 72 is padded to 80 by
//     the tensor map itself: d 0..63 land in a 128B-swizzled tile and d 64..79
//     in a 32B-swizzled tile, and d >= 72 lies outside the map so TMA fills
//     zeros.  The padding never exists in HBM;
//   * S = Q K^T runs as 5 tcgen05.mma (K = 16 each) into one of two TMEM
//     buffers, so the next tile's scores overlap this tile's softmax;
//   * the softmax warps keep a running max in the log2 domain and rescale O
//     (in TMEM) only when the max grows by more than 8, write P as bf16 into a
//     128B-swizzled shared tile, and the MMA warp accumulates O += P V with V
//     as an MN-major operand (two MMAs: N = 64 and N = 16);
//   * the epilogue divides by the row sum and stores bf16 O at column h*72.
#include "internal.h"
#include "ptx.cuh"

#include <cuda_fp16.h>

namespace vitq {
namespace {

constexpr int kBM = 128, kBN = 128, kStages = 3;
constexpr int kQLo = 0, kQHi = 16384;
constexpr int kKV0 = 20480, kKVStride = 40960;
constexpr int kKLo = 0, kKHi = 16384, kVLo = 20480, kVHi = 36864;
constexpr int kP = kKV0 + kStages * kKVStride;          // two 64-key atoms of 16 KB
constexpr int kBar = kP + 32768;
constexpr int kNumBars = 1 + 2 * kStages + 2 + 1 + 1;
constexpr size_t kAttnSmem = 1024 + kBar + kNumBars * 8 + 16;
constexpr uint32_t kTmemS = 0, kTmemO = 256;

struct AttnArgs {
  const int32_t* cu;
  __nv_bfloat16* out;
  int n_tokens;
  float scale_log2;
};

struct AttnSmem {
  uint8_t* base;
  __device__ uint32_t at(int off) const { return smem_u32(base + off); }
  __device__ uint64_t* bar(int i) const { return reinterpret_cast<uint64_t*>(base + kBar) + i; }
  __device__ uint32_t q_full() const { return smem_u32(bar(0)); }
  __device__ uint32_t kv_full(int s) const { return smem_u32(bar(1 + s)); }
  __device__ uint32_t kv_empty(int s) const { return smem_u32(bar(1 + kStages + s)); }
  __device__ uint32_t s_full(int b) const { return smem_u32(bar(1 + 2 * kStages + b)); }
  __device__ uint32_t p_full() const { return smem_u32(bar(3 + 2 * kStages)); }
  __device__ uint32_t pv_done() const { return smem_u32(bar(4 + 2 * kStages)); }
  __device__ uint32_t* tmem_holder() const { return reinterpret_cast<uint32_t*>(bar(kNumBars)); }
  __device__ volatile int* abort_flag() const {
    return reinterpret_cast<volatile int*>(tmem_holder() + 1);
  }
  __device__ uint32_t kv(int s, int part) const { return at(kKV0 + s * kKVStride + part); }
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ void attn_producer(const AttnSmem& sm, const CUtensorMap* tlo, const CUtensorMap* thi,
                              int head, int q_row, int kv_row0, int n_kv) {
  mbar_arrive_expect_tx(sm.q_full(), 20480);
  tma_load_3d(sm.at(kQLo), tlo, 0, head, q_row, sm.q_full());
  tma_load_3d(sm.at(kQHi), thi, 64, head, q_row, sm.q_full());
  for (int j = 0; j < n_kv; ++j) {
    const int s = j % kStages;
    const uint32_t ph = (uint32_t)(j / kStages) & 1u;
    if (!mbar_wait(sm.kv_empty(s), ph ^ 1u, sm.abort_flag())) return;
    mbar_arrive_expect_tx(sm.kv_full(s), 40960);
    const int row = kv_row0 + j * kBN;
    tma_load_3d(sm.kv(s, kKLo), tlo, 0, 16 + head, row, sm.kv_full(s));
    tma_load_3d(sm.kv(s, kKHi), thi, 64, 16 + head, row, sm.kv_full(s));
    tma_load_3d(sm.kv(s, kVLo), tlo, 0, 32 + head, row, sm.kv_full(s));
    tma_load_3d(sm.kv(s, kVHi), thi, 64, 32 + head, row, sm.kv_full(s));
  }
}

__device__ bool attn_issue_s(const AttnSmem& sm, uint32_t tmem, int j) {
  constexpr uint32_t idesc = make_idesc(1, 1, 0, 0, 128, 128);
  const int s = j % kStages;
  if (!mbar_wait(sm.kv_full(s), (uint32_t)(j / kStages) & 1u, sm.abort_flag())) return false;
  tc_fence_after();
  const uint32_t d = tmem + kTmemS + (uint32_t)(j & 1) * 128;
  const uint32_t qlo = sm.at(kQLo), klo = sm.kv(s, kKLo);
#pragma unroll
  for (int k = 0; k < 4; ++k)
    mma_bf16_ss(d, make_smem_desc(qlo + 32 * k, 16, 1024, kSwizzle128B),
                make_smem_desc(klo + 32 * k, 16, 1024, kSwizzle128B), idesc, k > 0 ? 1u : 0u);
  mma_bf16_ss(d, make_smem_desc(sm.at(kQHi), 16, 256, kSwizzle32B),
              make_smem_desc(sm.kv(s, kKHi), 16, 256, kSwizzle32B), idesc, 1u);
  tc_commit(sm.s_full(j & 1));
  return true;
}

template <bool kVF16>
__device__ void attn_mma(const AttnSmem& sm, uint32_t tmem, int n_kv) {
  // P.V operands: fp16 (format 0) when v was converted to fp16, else bf16 (format 1).
  constexpr uint32_t fmt = kVF16 ? 0u : 1u;
  constexpr uint32_t idesc_lo = make_idesc(fmt, fmt, 0, 1, 128, 64);
  constexpr uint32_t idesc_hi = make_idesc(fmt, fmt, 0, 1, 128, 16);
  if (!mbar_wait(sm.q_full(), 0, sm.abort_flag())) return;
  if (!attn_issue_s(sm, tmem, 0)) return;
  if (n_kv > 1 && !attn_issue_s(sm, tmem, 1)) return;
  const uint32_t p0 = sm.at(kP);
  for (int j = 0; j < n_kv; ++j) {
    if (!mbar_wait(sm.p_full(), (uint32_t)j & 1u, sm.abort_flag())) return;
    tc_fence_after();
    const int s = j % kStages;
    const uint32_t vlo = sm.kv(s, kVLo), vhi = sm.kv(s, kVHi);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint64_t ad = make_smem_desc(p0 + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024, kSwizzle128B);
      const uint32_t acc = (j > 0 || k > 0) ? 1u : 0u;
      mma_bf16_ss(tmem + kTmemO, ad, make_smem_desc(vlo + k * 2048, 16384, 1024, kSwizzle128B), idesc_lo,
                  acc);
      mma_bf16_ss(tmem + kTmemO + 64, ad, make_smem_desc(vhi + k * 512, 4096, 256, kSwizzle32B), idesc_hi,
                  acc);
    }
    tc_commit(sm.pv_done());
    tc_commit(sm.kv_empty(s));
    if (j + 2 < n_kv && !attn_issue_s(sm, tmem, j + 2)) return;
  }
}

__device__ __forceinline__ uint32_t pack_p(float lo, float hi, bool f16) {
  if (f16) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  return pack_bf16x2(lo, hi);
}

__device__ __forceinline__ float2 unpack_p(uint32_t u, bool f16) {
  if (f16) {
    __half2 h = *reinterpret_cast<__half2*>(&u);
    return __half22float2(h);
  }
  return unpack_bf16x2(u);
}

template <bool kVF16>
__device__ void attn_softmax(const AttnSmem& sm, uint32_t tmem, const AttnArgs& g, int head, int seq_start,
                             int seq_len, int q0, int n_kv) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quad = warp & 3;
  const int r = quad * 32 + lane;
  const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
  uint8_t* pbase = sm.base + kP;
  float m_run = -INFINITY, l_run = 0.f;
  for (int j = 0; j < n_kv; ++j) {
    bool ok = mbar_wait(sm.s_full(j & 1), (uint32_t)(j >> 1) & 1u, sm.abort_flag());
    if (!__all_sync(0xffffffffu, ok)) return;
    tc_fence_after();
    float sv[128];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t u[32];
      tmem_ld32(tmem + lane_addr + kTmemS + (uint32_t)(j & 1) * 128 + c * 32, u);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 32; ++i) sv[c * 32 + i] = __uint_as_float(u[i]);
    }
    const int valid = seq_len - j * kBN;
    if (valid < kBN) {
#pragma unroll
      for (int i = 0; i < 128; ++i)
        if (i >= valid) sv[i] = -INFINITY;
    }
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < 128; ++i) mx = fmaxf(mx, sv[i]);
    mx *= g.scale_log2;
    if (j > 0) {
      ok = mbar_wait(sm.pv_done(), (uint32_t)(j - 1) & 1u, sm.abort_flag());
      if (!__all_sync(0xffffffffu, ok)) return;
      tc_fence_after();
    }
    if (j == 0) {
      m_run = mx;
    } else {
      // tcgen05.ld/st are warp-collective: the whole warp rescales when any of
      // its rows needs it, with alpha = 1 for rows that keep their max.
      const bool need = mx > m_run + 8.f;
      if (__any_sync(0xffffffffu, need)) {
        const float m_new = need ? mx : m_run;
        const float alpha = ex2(m_run - m_new);
#pragma unroll
        for (int c = 0; c < 5; ++c) {
          uint32_t u[16];
          tmem_ld16(tmem + lane_addr + kTmemO + c * 16, u);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * alpha);
          tmem_st16(tmem + lane_addr + kTmemO + c * 16, u);
        }
        tmem_wait_st();
        l_run *= alpha;
        m_run = m_new;
      }
    }
    // P = 2^(s * scale_log2 - m_run), rounded to the P.V operand type, into the swizzled P tile.
    float lsum = 0.f;
#pragma unroll
    for (int a = 0; a < 2; ++a) {
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int k0 = a * 64 + c * 8 + 2 * i;
          const float p0 = ex2(fmaf(sv[k0], g.scale_log2, -m_run));
          const float p1 = ex2(fmaf(sv[k0 + 1], g.scale_log2, -m_run));
          w[i] = pack_p(p0, p1, kVF16);
          const float2 pr = unpack_p(w[i], kVF16);
          lsum += pr.x + pr.y;
        }
        uint8_t* dst = pbase + a * 16384 + r * 128 + ((c ^ (r & 7)) << 4);
        *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    l_run += lsum;
    fence_proxy_async_smem();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(sm.p_full());
  }
  bool ok = mbar_wait(sm.pv_done(), (uint32_t)(n_kv - 1) & 1u, sm.abort_flag());
  if (!__all_sync(0xffffffffu, ok)) return;
  tc_fence_after();
  float o[80];
#pragma unroll
  for (int c = 0; c < 5; ++c) {
    uint32_t u[16];
    tmem_ld16(tmem + lane_addr + kTmemO + c * 16, u);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 16; ++i) o[c * 16 + i] = __uint_as_float(u[i]);
  }
  if (q0 + r < seq_len && seq_start + q0 + r < g.n_tokens) {
    const float inv = 1.0f / l_run;
    __nv_bfloat16* dst = g.out + (size_t)(seq_start + q0 + r) * 1152 + head * 72;
#pragma unroll
    for (int c8 = 0; c8 < 9; ++c8) {
      uint4 u;
      u.x = pack_bf16x2(o[c8 * 8 + 0] * inv, o[c8 * 8 + 1] * inv);
      u.y = pack_bf16x2(o[c8 * 8 + 2] * inv, o[c8 * 8 + 3] * inv);
      u.z = pack_bf16x2(o[c8 * 8 + 4] * inv, o[c8 * 8 + 5] * inv);
      u.w = pack_bf16x2(o[c8 * 8 + 6] * inv, o[c8 * 8 + 7] * inv);
      *reinterpret_cast<uint4*>(dst + c8 * 8) = u;
    }
  }
}

template <bool kVF16>
__global__ void __launch_bounds__(192, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tlo, const __grid_constant__ CUtensorMap thi,
                const AttnArgs args) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const int qt = blockIdx.x, head = blockIdx.y, seq = blockIdx.z;
  const int seq_start = args.cu[seq];
  const int seq_len = args.cu[seq + 1] - seq_start;
  const int q0 = qt * kBM;
  if (q0 >= seq_len) return;
  const int n_kv = (seq_len + kBN - 1) / kBN;
  AttnSmem sm;
  sm.base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(sm.q_full(), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(sm.kv_full(s), 1);
      mbar_init(sm.kv_empty(s), 1);
    }
    mbar_init(sm.s_full(0), 1);
    mbar_init(sm.s_full(1), 1);
    mbar_init(sm.p_full(), 4);
    mbar_init(sm.pv_done(), 1);
    *sm.abort_flag() = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(sm.tmem_holder()), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sm.tmem_holder();
  if (warp == 0) {
    if (lane == 0) {
      prefetch_tensormap(&tlo);
      prefetch_tensormap(&thi);
      attn_producer(sm, &tlo, &thi, head, seq_start + q0, seq_start, n_kv);
    }
  } else if (warp == 1) {
    if (lane == 0) attn_mma<kVF16>(sm, tmem, n_kv);
  } else {
    attn_softmax<kVF16>(sm, tmem, args, head, seq_start, seq_len, q0, n_kv);
  }
  tc_fence_before();
  __syncthreads();
  if (*sm.abort_flag()) settle_pause(50000);
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_attention(const __nv_bfloat16* qkv, int n_tokens, const int32_t* cu, int n_seqs,
                             int max_seqlen, float scale, bool v_f16, __nv_bfloat16* out, cudaStream_t st) {
  if (n_tokens == 0 || n_seqs == 0 || max_seqlen == 0) return cudaSuccess;
  CUtensorMap tlo, thi;
  cudaError_t e = encode_tma_qkv(&tlo, qkv, n_tokens, 64, true);
  if (e != cudaSuccess) return e;
  e = encode_tma_qkv(&thi, qkv, n_tokens, 16, false);
  if (e != cudaSuccess) return e;
  auto kern = v_f16 ? attn_kernel<true> : attn_kernel<false>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kAttnSmem);
  if (e != cudaSuccess) return e;
  AttnArgs a{cu, out, n_tokens, scale * 1.4426950408889634f};
  dim3 grid((max_seqlen + kBM - 1) / kBM, 16, n_seqs);
  kern<<<grid, 192, kAttnSmem, st>>>(tlo, thi, a);
  return cudaGetLastError();
}

}  // namespace vitq
