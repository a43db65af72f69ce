// bf16 GEMM on the sm_100a tensor cores (tcgen05 kind::f16 + TMEM + TMA).
//
//   C[m, n] = bf16( sum_k A[m, k] W[n, k] + bias[n] + R[m, n] ),   fp32 accumulation
//
// "Qwen3-VL-8B on RTX 5090", section 4: the patch embedding, the first three
// ViT blocks and the mergers keep bf16 weights and activations (one massive
// activation channel makes the image embeddings sensitive to FP8 there).
//
// Design (B200): the FP8 GEMM's skeleton without the per-K-block promotion.
// There is one scale-free accumulation over all of K, so it stays in TMEM: the
// MMA thread accumulates a whole 128 x BN tile into one of two TMEM
// accumulators (tiles alternate), and the epilogue warps touch TMEM once per
// tile (bias, residual, bf16, staged in shared memory, TMA stores) while the
// next tile accumulates into the other one.
//   * warp 0: TMA producer, A and W tiles of 64 K-columns (128 bytes, 128B
//     swizzle, zero fill past M / N / K) into a multi-stage ring;
//   * warp 1: MMA issuer, 4 x tcgen05.mma kind::f16 (K = 16 each) per stage;
//   * BN/32 epilogue warps, thread = output row, 128 columns each.
#include "internal.h"
#include "ptx.cuh"

namespace vitq {
namespace {

template <int BN>
struct Bf16Cfg {
  static constexpr int BM = 128, BK = 64;   // BK bf16 = 128 bytes (one swizzle atom row)
  static constexpr int STAGES = BN == 256 ? 3 : 5;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int NACC = 2;            // TMEM accumulators (512 / BN >= 2)
  static constexpr int EPI_WARPS = BN / 32;
  static constexpr int EPI_WARP0 = BN == 256 ? 4 : 2;
  static constexpr int THREADS = BN == 256 ? 384 : 192;
  static constexpr int OUT_WARP_BYTES = 2 * 4096;   // two 64-column SW128 boxes of 32 rows
  static constexpr int OUT_BYTES = EPI_WARPS * (OUT_WARP_BYTES + 256);
  static constexpr int BAR_BYTES = (2 * STAGES + 2 * NACC + EPI_WARPS) * 8 + 16;
  static constexpr size_t SMEM = (size_t)STAGES * STAGE_BYTES + OUT_BYTES + 1024 + BAR_BYTES;
};

struct Bf16Args {
  const __nv_bfloat16* bias;
  const __nv_bfloat16* residual;
  int M, N, K;
};

template <int BN>
struct Bf16Smem {
  using Cfg = Bf16Cfg<BN>;
  uint8_t* base;
  __device__ uint32_t a(int s) const { return smem_u32(base + (size_t)s * Cfg::STAGE_BYTES); }
  __device__ uint32_t b(int s) const { return smem_u32(base + (size_t)s * Cfg::STAGE_BYTES + Cfg::A_BYTES); }
  __device__ uint8_t* out(int w) const {
    return base + (size_t)Cfg::STAGES * Cfg::STAGE_BYTES + (size_t)w * Cfg::OUT_WARP_BYTES;
  }
  __device__ uint8_t* bias(int w) const {
    return base + (size_t)Cfg::STAGES * Cfg::STAGE_BYTES + (size_t)Cfg::EPI_WARPS * Cfg::OUT_WARP_BYTES + w * 256;
  }
  __device__ uint64_t* bars() const {
    return reinterpret_cast<uint64_t*>(base + (size_t)Cfg::STAGES * Cfg::STAGE_BYTES + Cfg::OUT_BYTES);
  }
  __device__ uint32_t full(int s) const { return smem_u32(bars() + s); }
  __device__ uint32_t empty(int s) const { return smem_u32(bars() + Cfg::STAGES + s); }
  __device__ uint32_t tfull(int b) const { return smem_u32(bars() + 2 * Cfg::STAGES + b); }
  __device__ uint32_t tempty(int b) const { return smem_u32(bars() + 2 * Cfg::STAGES + Cfg::NACC + b); }
  __device__ uint32_t res_full(int w) const { return smem_u32(bars() + 2 * Cfg::STAGES + 2 * Cfg::NACC + w); }
  __device__ uint32_t* tmem_holder() const {
    return reinterpret_cast<uint32_t*>(bars() + 2 * Cfg::STAGES + 2 * Cfg::NACC + Cfg::EPI_WARPS);
  }
  __device__ volatile int* abort_flag() const { return reinterpret_cast<volatile int*>(tmem_holder() + 1); }
};

// Same tile order as the FP8 GEMM: m = t % tiles_m, n = (t / tiles_m + m) % tiles_n.
__device__ __forceinline__ void bf16_tile_coords(int tile, int tiles_m, int tiles_n, int& m, int& n) {
  m = tile % tiles_m;
  n = (tile / tiles_m + m) % tiles_n;
}

template <int BN>
__device__ void bf16_producer(const Bf16Smem<BN>& sm, const CUtensorMap* tmA, const CUtensorMap* tmB, int tiles_m,
                              int tiles_n, int num_tiles, int nkb) {
  using Cfg = Bf16Cfg<BN>;
  int stage = 0;
  uint32_t phase = 0;
  for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
    int mt, nt;
    bf16_tile_coords(tile, tiles_m, tiles_n, mt, nt);
    for (int kb = 0; kb < nkb; ++kb) {
      if (!mbar_wait(sm.empty(stage), phase ^ 1u, sm.abort_flag())) return;
      mbar_arrive_expect_tx(sm.full(stage), Cfg::STAGE_BYTES);
      tma_load_2d(sm.a(stage), tmA, kb * Cfg::BK, mt * Cfg::BM, sm.full(stage));
      tma_load_2d(sm.b(stage), tmB, kb * Cfg::BK, nt * BN, sm.full(stage));
      if (++stage == Cfg::STAGES) {
        stage = 0;
        phase ^= 1u;
      }
    }
  }
}

template <int BN>
__device__ void bf16_mma(const Bf16Smem<BN>& sm, uint32_t tmem_base, int num_tiles, int nkb) {
  using Cfg = Bf16Cfg<BN>;
  constexpr uint32_t idesc = make_idesc(1, 1, 0, 0, 128, BN);   // bf16 x bf16 -> fp32, both K-major
  int stage = 0;
  uint32_t phase = 0, it = 0;
  for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
    const uint32_t acc = it % Cfg::NACC;
    if (!mbar_wait(sm.tempty(acc), ((it / Cfg::NACC) & 1u) ^ 1u, sm.abort_flag())) return;
    tc_fence_after();
    for (int kb = 0; kb < nkb; ++kb) {
      if (!mbar_wait(sm.full(stage), phase, sm.abort_flag())) return;
      tc_fence_after();
      const uint32_t a0 = sm.a(stage), b0 = sm.b(stage);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        mma_bf16_ss(tmem_base + acc * BN, make_smem_desc(a0 + 32 * k, 16, 1024, kSwizzle128B),
                    make_smem_desc(b0 + 32 * k, 16, 1024, kSwizzle128B), idesc, (kb > 0 || k > 0) ? 1u : 0u);
      tc_commit(sm.empty(stage));
      if (++stage == Cfg::STAGES) {
        stage = 0;
        phase ^= 1u;
      }
    }
    tc_commit(sm.tfull(acc));
  }
}

template <int BN>
__device__ void bf16_epilogue(const Bf16Smem<BN>& sm, uint32_t tmem_base, const Bf16Args& g, const CUtensorMap* tmC,
                              const CUtensorMap* tmR, int tiles_m, int tiles_n, int num_tiles) {
  using Cfg = Bf16Cfg<BN>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quad = warp & 3;
  const int ew = warp - Cfg::EPI_WARP0;
  const int cg = ew >> 2;
  uint8_t* stg = sm.out(ew);
  const uint32_t stg_u32 = smem_u32(stg);
  uint8_t* bias_s = sm.bias(ew);
  const bool has_res = g.residual != nullptr;
  uint32_t it = 0;
  for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
    int mt, nt;
    bf16_tile_coords(tile, tiles_m, tiles_n, mt, nt);
    const int col0 = nt * BN + cg * 128;
    const int y0 = mt * Cfg::BM + quad * 32;
    const uint32_t acc = it % Cfg::NACC;
    // staging free (previous tile's stores read it), then residual by TMA and bias
    if (lane == 0) {
      bulk_wait_read_all();
      if (has_res) {
        mbar_arrive_expect_tx(sm.res_full(ew), Cfg::OUT_WARP_BYTES);
        tma_load_2d(stg_u32, tmR, col0, y0, sm.res_full(ew));
        tma_load_2d(stg_u32 + 4096, tmR, col0 + 64, y0, sm.res_full(ew));
      }
    }
    uint2 bias_l = make_uint2(0u, 0u);
    if (g.bias && col0 + 4 * lane < g.N) bias_l = __ldg(reinterpret_cast<const uint2*>(g.bias + col0 + 4 * lane));
    *reinterpret_cast<uint2*>(bias_s + lane * 8) = bias_l;
    __syncwarp();
    bool ok = mbar_wait(sm.tfull(acc), (it / Cfg::NACC) & 1u, sm.abort_flag());
    if (!__all_sync(0xffffffffu, ok)) return;
    if (has_res) {
      ok = mbar_wait(sm.res_full(ew), it & 1u, sm.abort_flag());
      if (!__all_sync(0xffffffffu, ok)) return;
    }
    tc_fence_after();
    const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + acc * BN + cg * 128;
#pragma unroll 1
    for (int c4 = 0; c4 < 4; ++c4) {   // 32 columns per TMEM round trip
      uint32_t r[32];
      tmem_ld32(taddr + c4 * 32, r);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int c8 = c4 * 4 + c;   // 8-column chunk 0..15
        const int h = c8 >> 3, cc = c8 & 7;
        float v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[c * 8 + i]);
        if (g.bias) {
          const uint4 bu = *reinterpret_cast<const uint4*>(bias_s + c8 * 16);
          const uint32_t bw[4] = {bu.x, bu.y, bu.z, bu.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = unpack_bf16x2(bw[i]);
            v[2 * i] += f.x;
            v[2 * i + 1] += f.y;
          }
        }
        uint4* slot = reinterpret_cast<uint4*>(stg + h * 4096 + lane * 128 + ((cc ^ (lane & 7)) << 4));
        if (has_res) {
          const uint4 ru = *slot;
          const uint32_t rw[4] = {ru.x, ru.y, ru.z, ru.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = unpack_bf16x2(rw[i]);
            v[2 * i] += f.x;
            v[2 * i + 1] += f.y;
          }
        }
        *slot = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                           pack_bf16x2(v[6], v[7]));
      }
    }
    // the accumulator is free for the tile after next
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(sm.tempty(acc));
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      if (y0 < g.M) {
        if (col0 < g.N) tma_store_2d(tmC, stg_u32, col0, y0);
        if (col0 + 64 < g.N) tma_store_2d(tmC, stg_u32 + 4096, col0 + 64, y0);
      }
      bulk_commit_group();
    }
  }
  if (lane == 0) bulk_wait_all();
}

template <int BN>
__global__ void __launch_bounds__(Bf16Cfg<BN>::THREADS, 1)
    bf16_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmR,
                     const Bf16Args args) {
  using Cfg = Bf16Cfg<BN>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  pdl_trigger();
  Bf16Smem<BN> sm;
  sm.base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nkb = (args.K + Cfg::BK - 1) / Cfg::BK;
  const int tiles_m = (args.M + Cfg::BM - 1) / Cfg::BM;
  const int tiles_n = (args.N + BN - 1) / BN;
  const int num_tiles = tiles_m * tiles_n;
  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::STAGES; ++s) {
      mbar_init(sm.full(s), 1);
      mbar_init(sm.empty(s), 1);
    }
    for (int b = 0; b < Cfg::NACC; ++b) {
      mbar_init(sm.tfull(b), 1);
      mbar_init(sm.tempty(b), Cfg::EPI_WARPS);
    }
    for (int w = 0; w < Cfg::EPI_WARPS; ++w) mbar_init(sm.res_full(w), 1);
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
  pdl_wait();   // inputs may be the previous kernel's outputs
  const uint32_t tmem_base = *sm.tmem_holder();
  if (warp < Cfg::EPI_WARP0) {
    if (warp == 0 && lane == 0) {
      prefetch_tensormap(&tmA);
      prefetch_tensormap(&tmB);
      bf16_producer<BN>(sm, &tmA, &tmB, tiles_m, tiles_n, num_tiles, nkb);
    } else if (warp == 1 && lane == 0) {
      bf16_mma<BN>(sm, tmem_base, num_tiles, nkb);
    }
  } else {
    bf16_epilogue<BN>(sm, tmem_base, args, &tmC, &tmR, tiles_m, tiles_n, num_tiles);
  }
  tc_fence_before();
  __syncthreads();
  if (*sm.abort_flag()) settle_pause(50000);
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

template <int BN>
cudaError_t bf16_launch_bn(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmC,
                           const CUtensorMap& tmR, const Bf16Args& a, int num_sms, cudaStream_t st) {
  using Cfg = Bf16Cfg<BN>;
  cudaError_t e = cudaFuncSetAttribute(bf16_gemm_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)Cfg::SMEM);
  if (e != cudaSuccess) return e;
  const int tiles = ((a.M + Cfg::BM - 1) / Cfg::BM) * ((a.N + BN - 1) / BN);
  const int grid = tiles < num_sms ? tiles : num_sms;
  return launch_pdl(bf16_gemm_kernel<BN>, dim3(grid), dim3(Cfg::THREADS), Cfg::SMEM, st, tmA, tmB, tmC, tmR, a);
}

}  // namespace

cudaError_t launch_bf16_gemm(const __nv_bfloat16* A, const __nv_bfloat16* W, const __nv_bfloat16* bias,
                             const __nv_bfloat16* residual, __nv_bfloat16* C, int M, int N, int K, int block_n,
                             int num_sms, cudaStream_t st) {
  if (M == 0 || N == 0) return cudaSuccess;
  CUtensorMap tmA, tmB, tmC, tmR;
  const int bn = block_n == 256 ? 256 : 128;
  cudaError_t e = encode_tma_2d_bf16(&tmA, A, K, M, 64, 128);
  if (e != cudaSuccess) return e;
  e = encode_tma_2d_bf16(&tmB, W, K, N, 64, bn);
  if (e != cudaSuccess) return e;
  e = encode_tma_2d_bf16(&tmC, C, N, M, 64, 32);
  if (e != cudaSuccess) return e;
  e = encode_tma_2d_bf16(&tmR, residual ? residual : C, N, M, 64, 32);
  if (e != cudaSuccess) return e;
  Bf16Args a{bias, residual, M, N, K};
  return bn == 256 ? bf16_launch_bn<256>(tmA, tmB, tmC, tmR, a, num_sms, st)
                   : bf16_launch_bn<128>(tmA, tmB, tmC, tmR, a, num_sms, st);
}

}  // namespace vitq
