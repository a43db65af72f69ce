// FP8 E4M3 W8A8 block-scaled GEMM on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
//   C[m, n] = bf16( sum_kb sA[kb, m] * sW[n / 128, kb] * (A_kb[m, :] . W_kb[n, :]) + bias[n] + R[m, n] )
//
// "Qwen3-VL-8B on RTX 5090", sections 1 and 3: the ViT linears run as FP8
// block-128 W8A8 GEMMs (per-token per-128-K activation scales, per-128x128
// weight scales), with the bias adds and the residual fused into the GEMM.
//
// Design (B200):
//   * persistent CTAs, one per SM, walking 128 x BN output tiles; or, with
//     kPair, clusters of two CTAs walking 256 x BN tiles: each CTA loads its
//     128 rows of A and half of the BN rows of W, and the leader issues
//     cta_group::2 MMAs that read both CTAs' shared memory and write both
//     CTAs' TMEM, so each SM fetches 16 + BN/2 x 128 bytes per K block instead
//     of 16 + BN x 128 (measured slower than single CTAs on the block's
//     shapes, so it is off unless VITQ_GEMM_PAIR=1);
//   * warp 0: TMA producer (A and W tiles of 128 K-columns into a multi-stage
//     128B-swizzled shared-memory ring, zero fill past K / M / N);
//   * warp 1: MMA issuer, 4 x tcgen05.mma kind::f8f6f4 (K = 32 each) per K
//     block into one of 512/BN TMEM partial buffers;
//   * BN/32 epilogue warps: each thread owns one output row and 128 columns,
//     reads the K block's partial from TMEM and accumulates
//     acc += partial * sA * sW in registers (the scales differ per K block, so
//     the tensor core cannot accumulate across K blocks); after the last K
//     block it adds bias and residual and writes bf16 into the warp's
//     128B-swizzled staging tile (32 rows x 128 columns), which one lane sends
//     to global memory with TMA stores.  The residual tile arrives by TMA into
//     the same staging tile while the K loop runs.  Row-per-thread global
//     stores (each a separate 16-byte sector) used to stall the next tile's
//     K loop for longer than the K loop itself.
#include "internal.h"
#include "ptx.cuh"

namespace vitq {
namespace {

// BN = 64: 6 warps (TMA, MMA, 4 epilogue warps, one per 32 rows); for small M.
// BN = 128: 10 warps (TMA, MMA, 8 epilogue warps, one per 64 columns x 32 rows).
// BN = 256: 12 warps
// (warpgroup 0 = TMA, MMA and two idle warps, which give registers away with
// setmaxnreg; warpgroups 1-2 = 8 epilogue warps, one per 128 columns x 32 rows).
#ifndef VITQ_SCALE_AHEAD
#define VITQ_SCALE_AHEAD 2
#endif

template <int BN, bool kPair = false>
struct GemmCfg {
  static constexpr int BM = 128, BK = 128;            // rows of A per CTA, K per stage
  static constexpr int TILE_M = kPair ? 256 : 128;    // rows per output tile
  static constexpr int B_ROWS = kPair ? BN / 2 : BN;  // rows of W loaded per CTA
  static constexpr int STAGES = kPair ? (BN == 256 ? 4 : 7) : (BN == 256 ? 3 : BN == 128 ? 5 : 7);
  static constexpr int A_BYTES = BM * BK;
  static constexpr int B_BYTES = B_ROWS * BK;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int NBUF = 512 / BN;
  // columns per epilogue warp: 64 for BN = 64 / 128 (4 / 8 epilogue warps: one TMEM
  // round trip per K block each), 128 for BN = 256 (the register file holds no more)
  static constexpr int COLS = BN == 256 ? 128 : 64;
  static constexpr int NH = COLS / 64;                // 64-column halves per warp
  static constexpr int EPI_WARPS = (BN / COLS) * 4;
  static constexpr int TEMPTY_COUNT = EPI_WARPS * (kPair ? 2 : 1);   // both CTAs' epilogues free a buffer
  // BN = 256 (single CTAs): warp 2 of warpgroup 0 (otherwise idle) stages each K
  // block's combined scales sA * sW for the tile's 128 rows and its two weight blocks
  // in a slot tied to the K block's TMEM buffer.  Otherwise each epilogue warp keeps
  // its 32 rows' activation scales of the next SA_DEPTH K blocks in its own ring (at
  // BN = 128 an extra scale warp measured slower: its K blocks are too short).
  static constexpr bool SCALE_WARP = BN == 256 && !kPair;
  static constexpr int SCALE_AHEAD = VITQ_SCALE_AHEAD;   // K blocks of scales in flight
  static constexpr int EPI_WARP0 = BN == 256 ? 4 : 2;
  static constexpr int THREADS = 32 * (EPI_WARP0 + EPI_WARPS);
  static constexpr bool SPLIT_REGS = BN == 256;
  static constexpr int MIN_LAUNCH_REGS = 168;   // 384 x 168 >= 128 x 56 + 256 x 224 (BN = 256)
  static constexpr int OUT_WARP_BYTES = NH * 4096;  // 64-column SW128 boxes of 32 rows
  static constexpr int OUT_BYTES = EPI_WARPS * (OUT_WARP_BYTES + COLS * 2);   // + the warp's bias values
  static constexpr int SA_DEPTH = 8;
  static constexpr int SA_BYTES = SCALE_WARP ? NBUF * (BN / 128) * 128 * 4 : EPI_WARPS * SA_DEPTH * 32 * 4;
  static constexpr int BAR_BYTES = (2 * STAGES + 2 * NBUF + EPI_WARPS) * 8 + 16;
  static constexpr size_t SMEM = (size_t)STAGES * STAGE_BYTES + OUT_BYTES + SA_BYTES + 1024 + BAR_BYTES;
};
static_assert(384 * GemmCfg<256>::MIN_LAUNCH_REGS >= 128 * 56 + 256 * 224, "register split");

struct GemmArgs {
  const float* sA;
  int ldsA;
  const float* sW;
  const __nv_bfloat16* bias;
  const __nv_bfloat16* residual;
  __nv_bfloat16* C;
  int M, N, K;
};

template <int BN, bool kPair>
struct GemmSmem {
  using Cfg = GemmCfg<BN, kPair>;
  uint8_t* base;
  __device__ uint32_t a(int s) const { return smem_u32(base + (size_t)s * Cfg::STAGE_BYTES); }
  __device__ uint32_t b(int s) const {
    return smem_u32(base + (size_t)s * Cfg::STAGE_BYTES + Cfg::A_BYTES);
  }
  __device__ uint8_t* out(int w) const {
    return base + (size_t)Cfg::STAGES * Cfg::STAGE_BYTES + (size_t)w * Cfg::OUT_WARP_BYTES;
  }
  __device__ uint8_t* bias(int w) const {
    return base + (size_t)Cfg::STAGES * Cfg::STAGE_BYTES + (size_t)Cfg::EPI_WARPS * Cfg::OUT_WARP_BYTES +
           w * Cfg::COLS * 2;
  }
  // combined scales of TMEM buffer b, weight block cb of the tile (128 rows, fp32)
  __device__ uint32_t scale_slot(int b, int cb) const {
    return smem_u32(base + (size_t)Cfg::STAGES * Cfg::STAGE_BYTES + Cfg::OUT_BYTES + (b * (BN / 128) + cb) * 512);
  }
  __device__ uint32_t sa_ring(int w) const {
    return smem_u32(base + (size_t)Cfg::STAGES * Cfg::STAGE_BYTES + Cfg::OUT_BYTES + w * Cfg::SA_DEPTH * 128);
  }
  __device__ uint64_t* bars() const {
    return reinterpret_cast<uint64_t*>(base + (size_t)Cfg::STAGES * Cfg::STAGE_BYTES + Cfg::OUT_BYTES +
                                       Cfg::SA_BYTES);
  }
  __device__ uint32_t full(int s) const { return smem_u32(bars() + s); }
  __device__ uint32_t empty(int s) const { return smem_u32(bars() + Cfg::STAGES + s); }
  __device__ uint32_t tfull(int b) const { return smem_u32(bars() + 2 * Cfg::STAGES + b); }
  __device__ uint32_t tempty(int b) const {
    return smem_u32(bars() + 2 * Cfg::STAGES + Cfg::NBUF + b);
  }
  __device__ uint32_t res_full(int w) const { return smem_u32(bars() + 2 * Cfg::STAGES + 2 * Cfg::NBUF + w); }
  __device__ uint32_t* tmem_holder() const {
    return reinterpret_cast<uint32_t*>(bars() + 2 * Cfg::STAGES + 2 * Cfg::NBUF + Cfg::EPI_WARPS);
  }
  __device__ volatile int* abort_flag() const {
    return reinterpret_cast<volatile int*>(tmem_holder() + 1);
  }
};

// Tile t -> (m, n): m = t % tiles_m, n = (t / tiles_m + m) % tiles_n.  A bijection
// on the tile grid in which the CTAs running at the same time read different W
// tiles (and each A tile is read by few of them), spreading the L2 traffic.
#ifndef VITQ_GEMM_DIAG
#define VITQ_GEMM_DIAG 1
#endif
__device__ __forceinline__ void tile_coords(int tile, int tiles_m, int tiles_n, int& m, int& n) {
  m = tile % tiles_m;
  const int q = tile / tiles_m;
  n = VITQ_GEMM_DIAG ? (q + m) % tiles_n : q;
}

// Tiles of this CTA (or CTA pair): t0, t0 + dt, ...
template <int BN, bool kPair>
__device__ void gemm_producer(const GemmSmem<BN, kPair>& sm, const CUtensorMap* tmA, const CUtensorMap* tmB,
                              int tiles_m, int tiles_n, int num_tiles, int nkb, int t0, int dt, int rank) {
  using Cfg = GemmCfg<BN, kPair>;
  int stage = 0;
  uint32_t phase = 0;
  for (int tile = t0; tile < num_tiles; tile += dt) {
    int mt, nt;
    tile_coords(tile, tiles_m, tiles_n, mt, nt);
    const int m0 = mt * Cfg::TILE_M + rank * Cfg::BM;
    const int n0 = nt * BN + rank * Cfg::B_ROWS;
    for (int kb = 0; kb < nkb; ++kb) {
      if (!mbar_wait(sm.empty(stage), phase ^ 1u, sm.abort_flag())) return;
      VITQ_TRACE_EV(1, (tile - t0) / dt * nkb + kb);  // producer: stage free, issuing loads
      if (kPair) {
        // both CTAs' copies count on the leader's full barrier, which expects them all
        const uint32_t full0 = mapa_shared(sm.full(stage), 0);
        if (rank == 0) mbar_arrive_expect_tx(sm.full(stage), 2 * Cfg::STAGE_BYTES);
        tma_load_2d_pair(sm.a(stage), tmA, kb * Cfg::BK, m0, full0);
        tma_load_2d_pair(sm.b(stage), tmB, kb * Cfg::BK, n0, full0);
      } else {
        mbar_arrive_expect_tx(sm.full(stage), Cfg::STAGE_BYTES);
        tma_load_2d(sm.a(stage), tmA, kb * Cfg::BK, m0, sm.full(stage));
        tma_load_2d(sm.b(stage), tmB, kb * Cfg::BK, n0, sm.full(stage));
      }
      if (++stage == Cfg::STAGES) {
        stage = 0;
        phase ^= 1u;
      }
    }
  }
}

template <int BN, bool kPair>
__device__ void gemm_mma(const GemmSmem<BN, kPair>& sm, uint32_t tmem_base, int num_tiles, int nkb, int t0,
                         int dt) {
  using Cfg = GemmCfg<BN, kPair>;
  constexpr uint32_t idesc = make_idesc(0, 0, 0, 0, Cfg::TILE_M, BN);
  int stage = 0;
  uint32_t phase = 0;
  uint32_t cnt = 0;
  for (int tile = t0; tile < num_tiles; tile += dt) {
    for (int kb = 0; kb < nkb; ++kb, ++cnt) {
      const uint32_t buf = cnt % Cfg::NBUF;
      const uint32_t aph = (cnt / Cfg::NBUF) & 1u;
      if (!mbar_wait(sm.tempty(buf), aph ^ 1u, sm.abort_flag())) return;
      tc_fence_after();
      VITQ_TRACE_EV(2, cnt);  // mma: TMEM buffer free
      if (!mbar_wait(sm.full(stage), phase, sm.abort_flag())) return;
      VITQ_TRACE_EV(3, cnt);  // mma: operands landed
      tc_fence_after();
      const uint32_t a0 = sm.a(stage), b0 = sm.b(stage);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint64_t ad = make_smem_desc(a0 + 32 * k, 16, 1024, kSwizzle128B);
        const uint64_t bd = make_smem_desc(b0 + 32 * k, 16, 1024, kSwizzle128B);
        if (kPair)
          mma_f8_ss_pair(tmem_base + buf * BN, ad, bd, idesc, k > 0 ? 1u : 0u);
        else
          mma_f8_ss(tmem_base + buf * BN, ad, bd, idesc, k > 0 ? 1u : 0u);
      }
      if (kPair) {   // release the stage in both CTAs; both epilogues may read their TMEM
        tc_commit_pair(sm.empty(stage), 0x3);
        tc_commit_pair(sm.tfull(buf), 0x3);
      } else {
        tc_commit(sm.empty(stage));
        tc_commit(sm.tfull(buf));
      }
      if (++stage == Cfg::STAGES) {
        stage = 0;
        phase ^= 1u;
      }
    }
  }
}

// Scale producer (BN = 256): for each K block of this CTA's tiles, in the
// MMA's order, sA[kb, m] * sW[n / 128, kb] for the tile's 128 rows and its weight
// blocks into the slot of the K block's TMEM buffer, once the epilogue has released
// that buffer (the tempty phase the MMA thread waits for); then one arrival on the
// buffer's tfull barrier, which completes when this and the MMAs' commit have both
// arrived.  Lane l handles rows 4l .. 4l + 3; the scales of the next SCALE_AHEAD
// K blocks are in flight in registers (a ring indexed by the unrolled loop).
template <int BN, bool kPair>
__device__ void gemm_scales(const GemmSmem<BN, kPair>& sm, const GemmArgs& g, int tiles_m, int tiles_n,
                            int num_tiles, int nkb, int t0, int dt) {
  using Cfg = GemmCfg<BN, kPair>;
  constexpr int WB = BN >= 128 ? BN / 128 : 1;   // weight blocks per tile
  constexpr int L = Cfg::SCALE_AHEAD;
  const int lane = threadIdx.x & 31;
  const int nbw = (g.N + 127) >> 7;   // weight blocks along N
  if (t0 >= num_tiles) return;
  const int total = ((num_tiles - t0 + dt - 1) / dt) * nkb;   // K blocks of this CTA
  int ltile = t0, lkb = 0;                                     // next K block to load
  auto load = [&](float (&a)[4], float (&w)[WB]) {
    int mt, nt;
    tile_coords(ltile, tiles_m, tiles_n, mt, nt);
    const int r0 = mt * Cfg::TILE_M + 4 * lane;
    const float* p = g.sA + (size_t)lkb * g.ldsA + r0;
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = r0 + i < g.M ? __ldg(p + i) : 0.f;
#pragma unroll
    for (int c = 0; c < WB; ++c) {
      const int nb = nt * WB + c;
      w[c] = nb < nbw ? __ldg(g.sW + (size_t)nb * nkb + lkb) : 0.f;
    }
    if (++lkb == nkb) {
      lkb = 0;
      ltile += dt;
    }
  };
  float a[L][4], w[L][WB];
#pragma unroll
  for (int j = 0; j < L; ++j)
    if (j < total) load(a[j], w[j]);
  for (int cnt = 0; cnt < total;) {
#pragma unroll
    for (int j = 0; j < L; ++j) {
      if (cnt < total) {
        const uint32_t buf = (uint32_t)cnt % Cfg::NBUF;
        const uint32_t aph = ((uint32_t)cnt / Cfg::NBUF) & 1u;
        if (!mbar_wait(sm.tempty(buf), aph ^ 1u, sm.abort_flag())) return;
#pragma unroll
        for (int c = 0; c < WB; ++c)
          st_shared_v4(sm.scale_slot(buf, c) + lane * 16, a[j][0] * w[j][c], a[j][1] * w[j][c], a[j][2] * w[j][c],
                       a[j][3] * w[j][c]);
        __syncwarp();
        if (lane == 0) mbar_arrive(sm.tfull(buf));   // release: the slot's stores come first
        if (cnt + L < total) load(a[j], w[j]);
        ++cnt;
      }
    }
  }
}

template <int BN, bool kPair>
__device__ void gemm_epilogue(const GemmSmem<BN, kPair>& sm, uint32_t tmem_base, const GemmArgs& g,
                              const CUtensorMap* tmC, const CUtensorMap* tmR, int tiles_m, int tiles_n,
                              int num_tiles, int nkb, int t0, int dt, int rank) {
  using Cfg = GemmCfg<BN, kPair>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quad = warp & 3;                         // TMEM lane quadrant this warp may access
  const int ew = warp - Cfg::EPI_WARP0;              // epilogue warp index
  const int cg = ew >> 2;                            // which COLS-column group of the tile
  const int r_in = quad * 32 + lane;
  uint8_t* stg = sm.out(ew);                         // staging: [NH boxes][32 rows][128 B], SW128
  const uint32_t stg_u32 = smem_u32(stg);
  const bool has_res = g.residual != nullptr;
  // the leader's tempty barriers count both CTAs' epilogue warps
  const uint32_t tempty0 = kPair ? mapa_shared(sm.tempty(0), 0) : sm.tempty(0);
  // Activation scales run SA_DEPTH - 1 K blocks ahead of their use through a ring
  // of SA_DEPTH slots in shared memory: each lane copies its own row's scale
  // (cp.async, zero past M), one group per K block, continuing into the next
  // tile's first K blocks, so a warp that falls behind the MMAs never waits for a
  // scale from L2.  A copy goes into the slot read one K block earlier.
  const uint32_t ring = sm.sa_ring(ew) + lane * 4;
  int pf_tile = t0, pf_kb = 0, pf_row = 0;
  auto pf_row_of = [&](int tile) {
    int mt_, nt_;
    tile_coords(tile, tiles_m, tiles_n, mt_, nt_);
    return mt_ * Cfg::TILE_M + rank * Cfg::BM + r_in;
  };
  if (pf_tile < num_tiles) pf_row = pf_row_of(pf_tile);
  uint32_t pf_q = 0;
  auto prefetch_scale = [&]() {
    if (pf_tile < num_tiles) {
      const bool in = pf_row < g.M;
      cp_async4(ring + (pf_q & (Cfg::SA_DEPTH - 1)) * 128, in ? g.sA + (size_t)pf_kb * g.ldsA + pf_row : g.sA,
                in ? 4u : 0u);
      if (++pf_kb == nkb) {
        pf_kb = 0;
        pf_tile += dt;
        if (pf_tile < num_tiles) pf_row = pf_row_of(pf_tile);
      }
    }
    cp_async_commit();
    ++pf_q;
  };
  if constexpr (!Cfg::SCALE_WARP) {
#pragma unroll 1
    for (int i = 0; i < Cfg::SA_DEPTH - 1; ++i) prefetch_scale();
  }
  uint32_t cnt = 0, it = 0;
  for (int tile = t0; tile < num_tiles; tile += dt, ++it) {
    int mt, nt;
    tile_coords(tile, tiles_m, tiles_n, mt, nt);
    const int m0 = mt * Cfg::TILE_M + rank * Cfg::BM;
    const int n0 = nt * BN;
    const int col0 = n0 + cg * Cfg::COLS;
    const int y0 = m0 + quad * 32;                   // first row of this warp's staging tile
    const bool col_ok = col0 < g.N;
    // this warp's COLS bias values (lane l: columns 4l..4l+3), loaded now and
    // parked in shared memory after the K loop
    uint2 bias_l = make_uint2(0u, 0u);
    if (g.bias && 4 * lane < Cfg::COLS && col0 + 4 * lane < g.N)
      bias_l = __ldg(reinterpret_cast<const uint2*>(g.bias + col0 + 4 * lane));
    // the residual tile is requested at the start of the tile, once the previous
    // tile's stores have read the staging tile
    if (has_res) {
      if (lane == 0) {
        bulk_wait_read_all();
        mbar_arrive_expect_tx(sm.res_full(ew), Cfg::OUT_WARP_BYTES);
#pragma unroll
        for (int h = 0; h < Cfg::NH; ++h) tma_load_2d(stg_u32 + h * 4096, tmR, col0 + h * 64, y0, sm.res_full(ew));
      }
      __syncwarp();
    }
    const float* sw_ptr = g.sW + (size_t)(col0 >> 7) * nkb;
    uint64_t acc[Cfg::NH * 32];
#pragma unroll
    for (int j = 0; j < Cfg::NH * 32; ++j) acc[j] = 0ull;
    // the weight scale (the same for the whole warp, an L1 hit) is loaded one K block ahead
    float sw_next = 0.f;
    if constexpr (!Cfg::SCALE_WARP) sw_next = col_ok ? __ldg(sw_ptr) : 0.f;
    for (int kb = 0; kb < nkb; ++kb, ++cnt) {
      const uint32_t buf = cnt % Cfg::NBUF;
      const uint32_t aph = (cnt / Cfg::NBUF) & 1u;
      float scale;
      if constexpr (!Cfg::SCALE_WARP) {
        cp_async_wait<Cfg::SA_DEPTH - 2>();
        scale = ld_shared_f32(ring + (cnt & (Cfg::SA_DEPTH - 1)) * 128) * sw_next;
        prefetch_scale();
        if (kb + 1 < nkb) sw_next = col_ok ? __ldg(sw_ptr + kb + 1) : 0.f;
      }
      if (lane == 0 && warp == Cfg::EPI_WARP0) VITQ_TRACE_EV(4, cnt);  // epilogue: waiting for partial
      const bool ok = mbar_wait(sm.tfull(buf), aph, sm.abort_flag());
      if (!__all_sync(0xffffffffu, ok)) return;
      // (with the scale warp, tfull also covers the scale slot)
      if constexpr (Cfg::SCALE_WARP)   // slot of this warp's weight block within the tile
        scale = ld_shared_f32(sm.scale_slot(buf, (cg * Cfg::COLS) >> 7) + r_in * 4);
      const uint64_t s2 = f2pack(scale, scale);
      if (lane == 0 && warp == Cfg::EPI_WARP0) VITQ_TRACE_EV(5, cnt);  // epilogue: partial ready
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + buf * BN + cg * Cfg::COLS;
#pragma unroll
      for (int h = 0; h < Cfg::NH; ++h) {
        uint32_t r0[32], r1[32];
        tmem_ld32(taddr + h * 64, r0);
        tmem_ld32(taddr + h * 64 + 32, r1);
        tmem_wait_ld();
        if (h == Cfg::NH - 1) {
          // the whole partial is in registers: the buffer goes back to the MMA
          // thread before the last FMAs, which keeps them off the hand-off chain
          tc_fence_before();
          __syncwarp();
          if (lane == 0 && warp == Cfg::EPI_WARP0) VITQ_TRACE_EV(6, cnt);  // epilogue: partial consumed
          if (lane == 0) {
            if (kPair)
              mbar_arrive_cluster(tempty0 + buf * 8);
            else
              mbar_arrive(sm.tempty(buf));
          }
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          acc[h * 32 + j] = ffma2(f2pack(__uint_as_float(r0[2 * j]), __uint_as_float(r0[2 * j + 1])), s2,
                                 acc[h * 32 + j]);
          acc[h * 32 + 16 + j] = ffma2(f2pack(__uint_as_float(r1[2 * j]), __uint_as_float(r1[2 * j + 1])), s2,
                                      acc[h * 32 + 16 + j]);
        }
      }
    }
    if (lane == 0 && warp == Cfg::EPI_WARP0) VITQ_TRACE_EV(7, it);  // epilogue: K loop done
    uint8_t* bias_s = sm.bias(ew);
    if (4 * lane < Cfg::COLS) *reinterpret_cast<uint2*>(bias_s + lane * 8) = bias_l;
    if (has_res) {
      const bool ok = mbar_wait(sm.res_full(ew), it & 1u, sm.abort_flag());
      if (!__all_sync(0xffffffffu, ok)) return;
    } else {
      if (lane == 0) bulk_wait_read_all();   // the previous tile's stores have read the staging tile
    }
    __syncwarp();
    if (lane == 0 && warp == Cfg::EPI_WARP0) VITQ_TRACE_EV(9, it);  // epilogue: staging free
    // bias + residual, bf16, into the staging tile (row = lane, 16-byte chunk c of
    // box h at position c ^ (lane & 7))
#pragma unroll
    for (int h = 0; h < Cfg::NH; ++h) {
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int c8 = h * 8 + c;
        float v[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = f2unpack(acc[c8 * 4 + i]);
          v[2 * i] = f.x;
          v[2 * i + 1] = f.y;
        }
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
        uint4* slot = reinterpret_cast<uint4*>(stg + h * 4096 + lane * 128 + ((c ^ (lane & 7)) << 4));
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
        uint4 o;
        o.x = pack_bf16x2(v[0], v[1]);
        o.y = pack_bf16x2(v[2], v[3]);
        o.z = pack_bf16x2(v[4], v[5]);
        o.w = pack_bf16x2(v[6], v[7]);
        *slot = o;
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0 && warp == Cfg::EPI_WARP0) VITQ_TRACE_EV(8, it);  // epilogue: staging written
    if (lane == 0) {
      // TMA clips rows >= M and columns >= N; boxes wholly outside are skipped
      if (y0 < g.M) {
#pragma unroll
        for (int h = 0; h < Cfg::NH; ++h)
          if (col0 + h * 64 < g.N) tma_store_2d(tmC, stg_u32 + h * 4096, col0 + h * 64, y0);
      }
      bulk_commit_group();
    }
  }
  if (lane == 0) bulk_wait_all();
}

template <int BN, bool kPair>
__global__ void __launch_bounds__(GemmCfg<BN, kPair>::THREADS, 1)
    fp8_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmR,
                    const GemmArgs args) {
  using Cfg = GemmCfg<BN, kPair>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  pdl_trigger();
  GemmSmem<BN, kPair> sm;
  sm.base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nkb = (args.K + Cfg::BK - 1) / Cfg::BK;
  const int tiles_m = (args.M + Cfg::TILE_M - 1) / Cfg::TILE_M;
  const int tiles_n = (args.N + BN - 1) / BN;
  const int num_tiles = tiles_m * tiles_n;
  // a CTA pair walks the tiles as one unit
  const int rank = kPair ? (int)cluster_ctarank() : 0;
  const int t0 = kPair ? (int)blockIdx.x / 2 : (int)blockIdx.x;
  const int dt = kPair ? (int)gridDim.x / 2 : (int)gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::STAGES; ++s) {
      mbar_init(sm.full(s), 1);
      mbar_init(sm.empty(s), 1);
    }
    for (int b = 0; b < Cfg::NBUF; ++b) {
      mbar_init(sm.tfull(b), Cfg::SCALE_WARP ? 2 : 1);   // MMA commit (+ scale warp)
      mbar_init(sm.tempty(b), Cfg::TEMPTY_COUNT);
    }
    for (int w = 0; w < Cfg::EPI_WARPS; ++w) mbar_init(sm.res_full(w), 1);
    *sm.abort_flag() = 0;
    fence_barrier_init();
  }
  if (kPair) cluster_sync_all();   // the peer's barriers exist before anything signals them
  if (warp == 1) {
    if (kPair) {
      tmem_alloc_pair(smem_u32(sm.tmem_holder()), 512);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(sm.tmem_holder()), 512);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();   // inputs may be the previous kernel's outputs
  const uint32_t tmem_base = *sm.tmem_holder();

  if (warp < Cfg::EPI_WARP0) {
    if (Cfg::SPLIT_REGS) asm volatile("setmaxnreg.dec.sync.aligned.u32 56;" ::: "memory");
    if (warp == 0 && lane == 0) {
      prefetch_tensormap(&tmA);
      prefetch_tensormap(&tmB);
      gemm_producer<BN, kPair>(sm, &tmA, &tmB, tiles_m, tiles_n, num_tiles, nkb, t0, dt, rank);
    } else if (warp == 1 && lane == 0 && rank == 0) {
      gemm_mma<BN, kPair>(sm, tmem_base, num_tiles, nkb, t0, dt);
    } else if (warp == 2) {
      if constexpr (Cfg::SCALE_WARP) gemm_scales<BN, kPair>(sm, args, tiles_m, tiles_n, num_tiles, nkb, t0, dt);
    }
  } else {
    if (Cfg::SPLIT_REGS) asm volatile("setmaxnreg.inc.sync.aligned.u32 224;" ::: "memory");
    gemm_epilogue<BN, kPair>(sm, tmem_base, args, &tmC, &tmR, tiles_m, tiles_n, num_tiles, nkb, t0, dt, rank);
  }

  tc_fence_before();
  __syncthreads();
  if (*sm.abort_flag()) settle_pause(50000);
  // neither CTA of a pair leaves while the leader's MMAs may still use the
  // peer's shared memory and TMEM (all of them completed before the last
  // partial was consumed by both epilogues)
  if (kPair) cluster_sync_all();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if (kPair)
      tmem_dealloc_pair(tmem_base, 512);
    else
      tmem_dealloc(tmem_base, 512);
  }
}

template <int BN, bool kPair>
cudaError_t launch_bn(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmC,
                      const CUtensorMap& tmR, const GemmArgs& a, int num_sms, cudaStream_t st) {
  using Cfg = GemmCfg<BN, kPair>;
  auto kern = fp8_gemm_kernel<BN, kPair>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::SMEM);
  if (e != cudaSuccess) return e;
  if (Cfg::SPLIT_REGS) {
    // setmaxnreg.inc only draws on the registers the CTA was launched with.
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    if (fa.numRegs < Cfg::MIN_LAUNCH_REGS) return cudaErrorInvalidConfiguration;
  }
  const int tiles = ((a.M + Cfg::TILE_M - 1) / Cfg::TILE_M) * ((a.N + BN - 1) / BN);
  if (!kPair) {
    const int grid = tiles < num_sms ? tiles : num_sms;
    return launch_pdl(kern, dim3(grid), dim3(Cfg::THREADS), Cfg::SMEM, st, tmA, tmB, tmC, tmR, a);
  }
  const int pairs = tiles < num_sms / 2 ? tiles : num_sms / 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(Cfg::THREADS, 1, 1);
  cfg.dynamicSmemBytes = Cfg::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, tmA, tmB, tmC, tmR, a);
}

}  // namespace

cudaError_t launch_fp8_gemm(const uint8_t* A, const float* sA, int ldsA, const uint8_t* W, const float* sW,
                            const __nv_bfloat16* bias, const __nv_bfloat16* residual, __nv_bfloat16* C,
                            int M, int N, int K, int block_n, bool pair, int num_sms, cudaStream_t st) {
  if (M == 0 || N == 0) return cudaSuccess;
  CUtensorMap tmA, tmB, tmC, tmR;
  const int bn = block_n == 256 ? 256 : (block_n == 64 && !pair) ? 64 : 128;
  cudaError_t e = encode_tma_2d_u8(&tmA, A, K, M, 128, 128);
  if (e != cudaSuccess) return e;
  e = encode_tma_2d_u8(&tmB, W, K, N, 128, pair ? bn / 2 : bn);
  if (e != cudaSuccess) return e;
  e = encode_tma_2d_bf16(&tmC, C, N, M, 64, 32);
  if (e != cudaSuccess) return e;
  e = encode_tma_2d_bf16(&tmR, residual ? residual : C, N, M, 64, 32);
  if (e != cudaSuccess) return e;
  GemmArgs a{sA, ldsA, sW, bias, residual, C, M, N, K};
  if (pair)
    return bn == 256 ? launch_bn<256, true>(tmA, tmB, tmC, tmR, a, num_sms, st)
                     : launch_bn<128, true>(tmA, tmB, tmC, tmR, a, num_sms, st);
  if (bn == 64) return launch_bn<64, false>(tmA, tmB, tmC, tmR, a, num_sms, st);
  return bn == 256 ? launch_bn<256, false>(tmA, tmB, tmC, tmR, a, num_sms, st)
                   : launch_bn<128, false>(tmA, tmB, tmC, tmR, a, num_sms, st);
}

}  // namespace vitq
