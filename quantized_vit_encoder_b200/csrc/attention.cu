// Block-diagonal non-causal attention over packed images, head_dim 72, on the
// sm_100a tensor cores.
//
// "Qwen3-VL-8B on RTX 5090", section 3 (FA2 full bidirectional attention per
// ViT block) and section 5 (each image is its own attention window, packed
// with cu_seqlens): O = softmax(Q K^T * scale) V per segment and head.
//
// Design (B200):
//   * one CTA per (segment, head, 256 queries = two 128-row Q tiles); 12 warps:
//     a TMA producer for K, one for V, one MMA issuer per Q tile, and four
//     softmax warps per Q tile, one per TMEM lane quadrant (thread = query row =
//     TMEM lane, owning all 128 score columns of its row, so the row max needs
//     no exchange between warps).  S_x(j+1) is computed while the softmax of
//     S_x(j) runs (the softmax frees S_x once it holds it in registers), and the
//     two tiles interleave on the tensor core;
//   * P is double-buffered per Q tile: the softmax writes P(j) into buffer j & 1
//     while P(j-1).V may still be reading the other one, and waits only for
//     P(j-2).V (per-buffer barriers, so no mbarrier phase can be confused with
//     the next);
//   * the softmax exponentials run on MUFU ex2; a share can move to a polynomial
//     on the FMA pipe (kPolyEvery).  The softmax warps of tile A and tile B that
//     share an SMSP may take turns for their exponentials (VITQ_ATTN_TURNS=1, off:
//     with two P buffers per tile both tiles' warps running at once is faster);
//   * K and V are read straight from the packed qkv activation [n, 3, 16, 72]
//     through 3D TMA maps (d, slot, token).  head_dim 72 is padded to 80 by
//     the tensor map itself: d >= 72 lies outside the map so TMA fills zeros,
//     and the padding never exists in HBM.  K (a ring of two stages): d 0..63 in
//     a 128B-swizzled tile, d 64..79 in a 32B-swizzled tile.  V (its own ring of
//     two stages): five 32B-swizzled atoms of 16 dims, so that P.V is one N = 80
//     MMA per 16 keys over 20 KB instead of two 64-wide 128B-swizzled atoms
//     (32 KB), which is what leaves room for the second P buffers.  A K stage is
//     freed by the S MMAs, a V stage by the P.V MMAs;
//   * the softmax threads copy their Q rows into TMEM once (columns packed two
//     bf16 per 32-bit column), and S = Q K^T runs as 5 tcgen05.mma with A in
//     TMEM (K = 16 each) into the tile's TMEM S buffer;
//   * the softmax warps keep a running max in the log2 domain and rescale O
//     (in TMEM) only when the max grows by more than 8, write P into a
//     128B-swizzled shared tile, and the MMA thread accumulates O += P V with
//     V as an MN-major operand;
//   * the epilogue divides by the row sum and stores bf16 O at column h*72.
#include "internal.h"
#include "ptx.cuh"

#include <cuda_fp16.h>

namespace vitq {
namespace {

constexpr int kBM = 128, kBN = 128, kQTiles = 2, kKStages = 2, kVStages = 2;
// Shared memory: a ring of K stages (d 0..63 in a 128B-swizzled tile, d 64..79 in a
// 32B-swizzled tile), a ring of V stages (five 32B-swizzled atoms of 16 dims, so
// that N = 80 spans them with one descriptor), and two P buffers per Q tile.
constexpr int kKStride = 20480, kKHi = 16384;
constexpr int kVStride = 20480, kVAtom = 4096;
constexpr int kK0 = 0, kV0 = kK0 + kKStages * kKStride;
constexpr int kP0 = kV0 + kVStages * kVStride;          // P buffer (x, b): two 64-key atoms of 16 KB
constexpr int kPBytes = 32768;
constexpr int kBar = kP0 + kQTiles * 2 * kPBytes;
// barriers: slot 0 (unused), k_full[2], k_empty[2], v_full[2], v_empty[2], s_full[2],
// s_free[2], p_full[2][2], pv_done[2][2] (per Q tile and P buffer), turn[2][4] (the
// softmax warp of tile x on SMSP q finished its exponentials), q_ready[2]
constexpr int kNumBars = 1 + 2 * kKStages + 2 * kVStages + 2 * kQTiles + 4 * kQTiles + kQTiles * 4 + kQTiles;
constexpr size_t kAttnSmem = 1024 + kBar + kNumBars * 8 + 16;
static_assert(kAttnSmem <= 232448, "shared memory budget");
// TMEM columns: S_A 0..127, S_B 128..255, O_A 256..335, Q_A 336..383, O_B 384..463,
// Q_B 464..511 (Q: 40 columns of bf16 pairs, written as 48).
__device__ __forceinline__ uint32_t tmem_s(int x) { return (uint32_t)x * 128u; }
__device__ __forceinline__ uint32_t tmem_o(int x) { return 256u + (uint32_t)x * 128u; }
__device__ __forceinline__ uint32_t tmem_q(int x) { return 336u + (uint32_t)x * 128u; }
// Warpgroup 0: warp 0 the K producer, warps 1 and 2 the MMA issuers for Q tiles A
// and B, warp 3 the V producer; warps 4-7 the softmax of Q tile A, 8-11 of Q tile B
// (one per TMEM lane quadrant).
constexpr int kThreads = 128 + 128 * kQTiles;
// register split: warpgroup 0 (TMA, MMA) 56 per thread, the softmax warpgroups 208
constexpr int kAttnMinLaunchRegs = 158;
static_assert(kThreads * kAttnMinLaunchRegs >= 128 * 56 + 256 * 208, "register split");
// Share of the softmax exponentials moved from MUFU to the FMA-pipe polynomial:
// one pair in kPolyEvery (0 = none).  MUFU ex2 runs at 16 per clock per SM.
#ifndef VITQ_ATTN_POLY_EVERY
#define VITQ_ATTN_POLY_EVERY 0
#endif
constexpr int kPolyEvery = VITQ_ATTN_POLY_EVERY;
constexpr int kPolyMod = kPolyEvery > 0 ? kPolyEvery : 1;
// 8-key group of the exponential loop (16 per step) after which the turn passes to the other tile (15 = at the end).
#ifndef VITQ_ATTN_TURN_AT
#define VITQ_ATTN_TURN_AT 11
#endif
constexpr int kTurnAt = VITQ_ATTN_TURN_AT;
// Whether the two tiles' softmax warps of one SMSP take turns for the exponentials
// (with two P buffers per tile the turns measured slower: 278 vs 271 us at 6256 tokens).
#ifndef VITQ_ATTN_TURNS
#define VITQ_ATTN_TURNS 0
#endif
constexpr bool kTakeTurns = VITQ_ATTN_TURNS != 0;

struct AttnArgs {
  const __nv_bfloat16* qkv;
  const int32_t* cu;
  __nv_bfloat16* out;
  int n_tokens;
  float scale_log2;
};

// K/V tiles are visited starting at a per-CTA offset so that the CTAs of one
// head, which run at the same time, read different K/V tiles (online softmax
// does not depend on the order).  The offset depends only on the Q-tile index
// within its segment, so a segment gives the same result packed or alone.
#ifndef VITQ_ATTN_STAGGER
#define VITQ_ATTN_STAGGER 1
#endif
__device__ __forceinline__ int kv_tile(int j, int off, int n_kv) {
  const int t = j + off;
  return t >= n_kv ? t - n_kv : t;
}

struct AttnSmem {
  uint8_t* base;
  __device__ uint32_t at(int off) const { return smem_u32(base + off); }
  __device__ uint64_t* bar(int i) const { return reinterpret_cast<uint64_t*>(base + kBar) + i; }
  __device__ uint32_t k_full(int s) const { return smem_u32(bar(1 + s)); }
  __device__ uint32_t k_empty(int s) const { return smem_u32(bar(1 + kKStages + s)); }
  __device__ uint32_t v_full(int s) const { return smem_u32(bar(1 + 2 * kKStages + s)); }
  __device__ uint32_t v_empty(int s) const { return smem_u32(bar(1 + 2 * kKStages + kVStages + s)); }
  static constexpr int kB0 = 1 + 2 * kKStages + 2 * kVStages;
  __device__ uint32_t s_full(int x) const { return smem_u32(bar(kB0 + x)); }
  __device__ uint32_t s_free(int x) const { return smem_u32(bar(kB0 + kQTiles + x)); }
  __device__ uint32_t p_full(int x, int b) const { return smem_u32(bar(kB0 + 2 * kQTiles + x * 2 + b)); }
  __device__ uint32_t pv_done(int x, int b) const { return smem_u32(bar(kB0 + 4 * kQTiles + x * 2 + b)); }
  __device__ uint32_t turn(int x, int q) const { return smem_u32(bar(kB0 + 6 * kQTiles + x * 4 + q)); }
  __device__ uint32_t q_ready(int x) const { return smem_u32(bar(kB0 + 10 * kQTiles + x)); }
  __device__ uint32_t* tmem_holder() const { return reinterpret_cast<uint32_t*>(bar(kNumBars)); }
  __device__ volatile int* abort_flag() const {
    return reinterpret_cast<volatile int*>(tmem_holder() + 1);
  }
  __device__ uint32_t k(int s) const { return at(kK0 + s * kKStride); }
  __device__ uint32_t v(int s) const { return at(kV0 + s * kVStride); }
  __device__ uint32_t p(int x, int b) const { return at(kP0 + (x * 2 + b) * kPBytes); }
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA/ALU pipes for a pair of values (Cody-Waite split x = n + f,
// |f| <= 1/2, then a degree-3 polynomial fitted to 2^f on [-1/2, 1/2]: max
// relative error 7.5e-5, below the fp16 rounding of P).  n is read from the low
// bits of x + 1.5*2^23 and added to the exponent field; x is clamped at -125
// (2^-125 is 0 once P is rounded).
// ex2_poly on a pair of values with packed fp32 arithmetic.
__device__ __forceinline__ float2 ex2_poly2(float x0, float x1) {
  const uint64_t magic = f2pack(12582912.0f, 12582912.0f), nmagic = f2pack(-12582912.0f, -12582912.0f);
  const uint64_t x = f2pack(fmaxf(x0, -125.0f), fmaxf(x1, -125.0f));
  const uint64_t j = fadd2(x, magic);
  const uint64_t f = ffma2(fadd2(j, nmagic), f2pack(-1.0f, -1.0f), x);
  uint64_t p = ffma2(f2pack(0.0551716648f, 0.0551716648f), f, f2pack(0.2426111251f, 0.2426111251f));
  p = ffma2(p, f, f2pack(0.6932609677f, 0.6932609677f));
  p = ffma2(p, f, f2pack(0.9999280572f, 0.9999280572f));
  const float2 pp = f2unpack(p), jj = f2unpack(j);
  return make_float2(__int_as_float(__float_as_int(pp.x) + (__float_as_int(jj.x) << 23)),
                     __int_as_float(__float_as_int(pp.y) + (__float_as_int(jj.y) << 23)));
}



// K tiles (warp 0) and V tiles (warp 3) come from the packed qkv activation
// through 3D maps (d, slot, token); d >= 72 lies outside the map and reads zero.
// A K stage is free once both tiles' S MMAs of it have completed, a V stage once
// both tiles' P.V MMAs have.
__device__ void attn_load_k(const AttnSmem& sm, const CUtensorMap* tlo, const CUtensorMap* thi, int head,
                            int kv_row0, int n_kv, int off) {
  for (int j = 0; j < n_kv; ++j) {
    const int s = j % kKStages;
    const uint32_t ph = (uint32_t)(j / kKStages) & 1u;
    if (!mbar_wait(sm.k_empty(s), ph ^ 1u, sm.abort_flag())) return;
    mbar_arrive_expect_tx(sm.k_full(s), kKStride);
    const int row = kv_row0 + kv_tile(j, off, n_kv) * kBN;
    tma_load_3d(sm.k(s), tlo, 0, 16 + head, row, sm.k_full(s));
    tma_load_3d(sm.k(s) + kKHi, thi, 64, 16 + head, row, sm.k_full(s));
  }
}
__device__ void attn_load_v(const AttnSmem& sm, const CUtensorMap* thi, int head, int kv_row0, int n_kv,
                            int off) {
  for (int j = 0; j < n_kv; ++j) {
    const int s = j % kVStages;
    const uint32_t ph = (uint32_t)(j / kVStages) & 1u;
    if (!mbar_wait(sm.v_empty(s), ph ^ 1u, sm.abort_flag())) return;
    mbar_arrive_expect_tx(sm.v_full(s), kVStride);
    const int row = kv_row0 + kv_tile(j, off, n_kv) * kBN;
#pragma unroll
    for (int a = 0; a < 5; ++a) tma_load_3d(sm.v(s) + a * kVAtom, thi, 16 * a, 32 + head, row, sm.v_full(s));
  }
}

// S_x = Q_x K_j^T (5 MMAs of K = 16 over the padded head_dim 80, Q from TMEM) into S buffer x.
__device__ bool attn_issue_s(const AttnSmem& sm, uint32_t tmem, int x, int j) {
  constexpr uint32_t idesc = make_idesc(1, 1, 0, 0, 128, 128);
  const int s = j % kKStages;
  if (!mbar_wait(sm.k_full(s), (uint32_t)(j / kKStages) & 1u, sm.abort_flag())) return false;
  tc_fence_after();
  const uint32_t d = tmem + tmem_s(x), q = tmem + tmem_q(x);
  const uint32_t klo = sm.k(s);
#pragma unroll
  for (int k = 0; k < 4; ++k)
    mma_bf16_ts(d, q + 8 * k, make_smem_desc(klo + 32 * k, 16, 1024, kSwizzle128B), idesc, k > 0 ? 1u : 0u);
  mma_bf16_ts(d, q + 32, make_smem_desc(klo + kKHi, 16, 256, kSwizzle32B), idesc, 1u);
  tc_commit(sm.s_full(x));
  tc_commit(sm.k_empty(s));
  return true;
}

// O_x += P_x(j) V_j: P from shared memory (K-major, buffer j & 1), V MN-major in
// five 16-wide 32B-swizzled atoms (LBO 4096 bytes apart); one N = 80 MMA per 16 keys.
template <bool kVF16>
__device__ bool attn_issue_pv(const AttnSmem& sm, uint32_t tmem, int x, int j) {
  constexpr uint32_t fmt = kVF16 ? 0u : 1u;
  constexpr uint32_t idesc = make_idesc(fmt, fmt, 0, 1, 128, 80);
  const int b = j & 1;
  if (!mbar_wait(sm.p_full(x, b), (uint32_t)(j >> 1) & 1u, sm.abort_flag())) return false;
  const int s = j % kVStages;
  if (!mbar_wait(sm.v_full(s), (uint32_t)(j / kVStages) & 1u, sm.abort_flag())) return false;
  VITQ_TRACE_EV(14 + x, j);   // mma: P complete
  tc_fence_after();
  const uint32_t vb = sm.v(s), p0 = sm.p(x, b);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint64_t ad = make_smem_desc(p0 + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024, kSwizzle128B);
    const uint32_t acc = (j > 0 || k > 0) ? 1u : 0u;
    mma_bf16_ss(tmem + tmem_o(x), ad, make_smem_desc(vb + k * 512, kVAtom, 256, kSwizzle32B), idesc, acc);
  }
  tc_commit(sm.pv_done(x, b));
  tc_commit(sm.v_empty(s));
  return true;
}

// Tensor-core work of Q tile x, issued by its own thread.  S_x(j+1) is issued as
// soon as the softmax has moved S_x(j) into registers (s_free), so it overlaps
// that softmax; P_x(j).V_j follows when P_x(j) is in shared memory.
template <bool kVF16>
__device__ void attn_mma(const AttnSmem& sm, uint32_t tmem, int x, int n_kv) {
  if (!mbar_wait(sm.q_ready(x), 0, sm.abort_flag())) return;
  tc_fence_after();
  if (!attn_issue_s(sm, tmem, x, 0)) return;
  for (int j = 0; j < n_kv; ++j) {
    if (j + 1 < n_kv) {
      if (!mbar_wait(sm.s_free(x), (uint32_t)j & 1u, sm.abort_flag())) return;
      VITQ_TRACE_EV(16 + x, j);   // mma: S buffer free
      tc_fence_after();
      if (!attn_issue_s(sm, tmem, x, j + 1)) return;
      VITQ_TRACE_EV(10 + x, j + 1);   // mma: S issued
    }
    if (!attn_issue_pv<kVF16>(sm, tmem, x, j)) return;
    VITQ_TRACE_EV(12 + x, j);     // mma: P.V issued
  }
}

__device__ __forceinline__ uint32_t pack_p(float lo, float hi, bool f16) {
  if (f16) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  return pack_bf16x2(lo, hi);
}

// One warp per (Q tile, TMEM lane quadrant); thread = query row = TMEM lane,
// owning all 128 score columns of its row, so the row max needs no exchange
// between warps.  The warp copies its Q rows into TMEM, rescales its O rows and
// writes their output.
template <bool kVF16>
__device__ void attn_softmax(const AttnSmem& sm, uint32_t tmem, const AttnArgs& g, int x, int n_q,
                             int head, int seq_start, int seq_len, int q0, int n_kv, int off) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quad = warp & 3;
  const int r = quad * 32 + lane;
  const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
  const uint32_t s_addr = tmem + lane_addr + tmem_s(x), o_addr = tmem + lane_addr + tmem_o(x);
  uint8_t* pbase0 = sm.base + kP0 + x * 2 * kPBytes;
  const bool tr = quad == 0 && lane == 0;
  (void)tr;
  {
    // this thread's Q row -> TMEM (bf16 pairs in columns 0..35, zeros up to 47)
    const bool q_ok = q0 + r < seq_len && seq_start + q0 + r < g.n_tokens;
    const uint4* src = reinterpret_cast<const uint4*>(g.qkv + (size_t)(seq_start + q0 + r) * 3456 + head * 72);
    const uint32_t q_addr = tmem + lane_addr + tmem_q(x);
#pragma unroll
    for (int c = 0; c < 3; ++c) {
      uint32_t qw[16];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 v = (q_ok && c * 4 + i < 9) ? __ldg(src + c * 4 + i) : make_uint4(0u, 0u, 0u, 0u);
        qw[i * 4 + 0] = v.x;
        qw[i * 4 + 1] = v.y;
        qw[i * 4 + 2] = v.z;
        qw[i * 4 + 3] = v.w;
      }
      tmem_st16(q_addr + c * 16, qw);
    }
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(sm.q_ready(x));
  }
  float m_run = -INFINITY, l_run = 0.f;
  for (int j = 0; j < n_kv; ++j) {
    bool ok = mbar_wait(sm.s_full(x), (uint32_t)j & 1u, sm.abort_flag());
    if (!__all_sync(0xffffffffu, ok)) return;
    if (tr) VITQ_TRACE_EV(20 + x, j);   // softmax: S ready
    tc_fence_after();
    // keys of this tile inside the segment
    const int valid = seq_len - kv_tile(j, off, n_kv) * kBN;
    uint32_t su[4][32];
    tmem_ld32(s_addr, su[0]);
    tmem_ld32(s_addr + 32, su[1]);
    tmem_ld32(s_addr + 64, su[2]);
    tmem_ld32(s_addr + 96, su[3]);
    tmem_wait_ld();
    if (tr) VITQ_TRACE_EV(26 + x, j);   // softmax: S in registers
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(sm.s_free(x));
    if (valid < kBN) {
#pragma unroll
      for (int i = 0; i < kBN; ++i)
        if (i >= valid) su[i >> 5][i & 31] = 0xFF800000u;   // -inf
    }
    // row max: 8 independent chains of 3-input max, then a tree
    float mp[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) mp[k] = __uint_as_float(su[0][k]);
#pragma unroll
    for (int i = 8; i < kBN; i += 16)
#pragma unroll
      for (int k = 0; k < 8; ++k)
        mp[k] = fmax3(mp[k], __uint_as_float(su[(i + k) >> 5][(i + k) & 31]),
                      __uint_as_float(su[(i + 8 + k) >> 5][(i + 8 + k) & 31]));
    const float mx = fmax3(fmax3(mp[0], mp[1], mp[2]), fmax3(mp[3], mp[4], mp[5]), fmaxf(mp[6], mp[7])) *
                     g.scale_log2;
    // P(j) goes to buffer j & 1, which P(j-2).V must have finished reading
    const int pb = j & 1;
    uint8_t* pbase = pbase0 + pb * kPBytes;
    if (j >= 2) {
      ok = mbar_wait(sm.pv_done(x, pb), (uint32_t)((j - 2) >> 1) & 1u, sm.abort_flag());
      if (!__all_sync(0xffffffffu, ok)) return;
      tc_fence_after();
    }
    if (tr) VITQ_TRACE_EV(22 + x, j);   // softmax: max known, O stable
    // new running max: it changes only when the tile max exceeds it by more than 8
    // (so P <= 2^8), and the decision is warp-uniform because the O rescale uses
    // warp-collective tcgen05.ld/st (rows that keep their max get alpha = 1).
    float alpha = 1.f;
    bool rescale = false;
    if (j == 0) {
      m_run = mx;
    } else {
      const bool need = mx > m_run + 8.f;
      rescale = __any_sync(0xffffffffu, need);
      if (need) {
        alpha = ex2(m_run - mx);
        m_run = mx;
      }
    }
    // The softmax warps of the two tiles on one SMSP take turns for the
    // exponentials (A(j), B(j), A(j+1), ...): MUFU serves one tile at full rate
    // while the other reads its next scores and waits for its P.V.
    if (kTakeTurns && n_q == 2 && (x == 1 || j > 0)) {
      ok = mbar_wait(sm.turn(1 - x, quad), (uint32_t)(x == 1 ? j : j - 1) & 1u, sm.abort_flag());
      if (!__all_sync(0xffffffffu, ok)) return;
    }
    if (tr) VITQ_TRACE_EV(28 + x, j);   // softmax: turn for the exponentials
    // P = 2^(s * scale_log2 - m_run), rounded to the P.V operand type, into the
    // two 64-key atoms of the swizzled P tile; 8 fp32 partial row sums.
    const uint64_t sc2 = f2pack(g.scale_log2, g.scale_log2), nm2 = f2pack(-m_run, -m_run);
    uint64_t ls[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
    for (int c = 0; c < kBN / 8; ++c) {
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int k0 = c * 8 + 2 * i;
        const float2 t = f2unpack(ffma2(f2pack(__uint_as_float(su[k0 >> 5][k0 & 31]),
                                               __uint_as_float(su[(k0 + 1) >> 5][(k0 + 1) & 31])),
                                        sc2, nm2));
        float2 p;
        if (kPolyEvery > 0 && (i % kPolyMod) == kPolyMod - 1) {
          p = ex2_poly2(t.x, t.y);
        } else {
          p.x = ex2(t.x);
          p.y = ex2(t.y);
        }
        w[i] = pack_p(p.x, p.y, kVF16);
        ls[i] = fadd2(ls[i], f2pack(p.x, p.y));
      }
      uint8_t* dst = pbase + (c >> 3) * 16384 + r * 128 + (((c & 7) ^ (r & 7)) << 4);
      *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
      // hand the turn to the other tile a little before the end, so that its
      // exponentials start while these finish (hides the hand-over latency)
      if (kTakeTurns && c == kTurnAt && n_q == 2 && !(x == 1 && j == n_kv - 1)) {
        __syncwarp();
        if (lane == 0) mbar_arrive(sm.turn(x, quad));
      }
    }
    if (rescale) {
      // O to the new max once P.V(j-1) has completed (it is read and written here);
      // done after P so the scores are dead
      ok = mbar_wait(sm.pv_done(x, (j - 1) & 1), (uint32_t)((j - 1) >> 1) & 1u, sm.abort_flag());
      if (!__all_sync(0xffffffffu, ok)) return;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < 5; ++c) {
        uint32_t u[16];
        tmem_ld16(o_addr + c * 16, u);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * alpha);
        tmem_st16(o_addr + c * 16, u);
      }
      tmem_wait_st();
    }
    {
      const float2 l0 = f2unpack(fadd2(ls[0], ls[1])), l1 = f2unpack(fadd2(ls[2], ls[3]));
      l_run = l_run * alpha + ((l0.x + l0.y) + (l1.x + l1.y));
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncwarp();
    if (tr) VITQ_TRACE_EV(24 + x, j);   // softmax: P written
    if (lane == 0) mbar_arrive(sm.p_full(x, pb));
  }
  // the last P.V's commit tracks every earlier MMA of the tile
  bool ok = mbar_wait(sm.pv_done(x, (n_kv - 1) & 1), (uint32_t)((n_kv - 1) >> 1) & 1u, sm.abort_flag());
  if (!__all_sync(0xffffffffu, ok)) return;
  tc_fence_after();
  const float l_sum = l_run;
  // O / l in 16-column chunks (columns 72..79 are the zero padding and are not stored)
  const bool row_ok = q0 + r < seq_len && seq_start + q0 + r < g.n_tokens;
  const float inv = 1.0f / l_sum;
  __nv_bfloat16* dst = g.out + (size_t)(seq_start + q0 + r) * 1152 + head * 72;
#pragma unroll
  for (int c = 0; c < 5; ++c) {
    uint32_t u[16];
    tmem_ld16(o_addr + c * 16, u);
    tmem_wait_ld();
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      if (row_ok && c * 2 + hh < 9) {
        uint4 v;
        v.x = pack_bf16x2(__uint_as_float(u[hh * 8 + 0]) * inv, __uint_as_float(u[hh * 8 + 1]) * inv);
        v.y = pack_bf16x2(__uint_as_float(u[hh * 8 + 2]) * inv, __uint_as_float(u[hh * 8 + 3]) * inv);
        v.z = pack_bf16x2(__uint_as_float(u[hh * 8 + 4]) * inv, __uint_as_float(u[hh * 8 + 5]) * inv);
        v.w = pack_bf16x2(__uint_as_float(u[hh * 8 + 6]) * inv, __uint_as_float(u[hh * 8 + 7]) * inv);
        *reinterpret_cast<uint4*>(dst + (c * 2 + hh) * 8) = v;
      }
    }
  }
}

template <bool kVF16>
__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tlo, const __grid_constant__ CUtensorMap thi,
                const AttnArgs args) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  pdl_trigger();
  const int head = blockIdx.y, seq = blockIdx.z;
  const int seq_start = args.cu[seq];
  const int seq_len = args.cu[seq + 1] - seq_start;
  const int q0 = blockIdx.x * kBM * kQTiles;
  if (q0 >= seq_len) return;
  const int n_q = (seq_len - q0) > kBM ? kQTiles : 1;   // Q tiles of this CTA that hold rows
  const int n_kv = (seq_len + kBN - 1) / kBN;
  const int off = VITQ_ATTN_STAGGER ? (int)((blockIdx.x * 7u) % (unsigned)n_kv) : 0;
  AttnSmem sm;
  sm.base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(sm.k_full(s), 1);
      mbar_init(sm.k_empty(s), (uint32_t)n_q);       // one commit per active Q tile
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(sm.v_full(s), 1);
      mbar_init(sm.v_empty(s), (uint32_t)n_q);
    }
    for (int x = 0; x < kQTiles; ++x) {
      for (int q = 0; q < 4; ++q) mbar_init(sm.turn(x, q), 1);
      mbar_init(sm.q_ready(x), 4);
      mbar_init(sm.s_full(x), 1);
      mbar_init(sm.s_free(x), 4);
      for (int b = 0; b < 2; ++b) {
        mbar_init(sm.p_full(x, b), 4);
        mbar_init(sm.pv_done(x, b), 1);
      }
    }
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
  const uint32_t tmem = *sm.tmem_holder();
  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 56;" ::: "memory");
    if (warp == 0 && lane == 0) {
      prefetch_tensormap(&tlo);
      prefetch_tensormap(&thi);
      attn_load_k(sm, &tlo, &thi, head, seq_start, n_kv, off);
    } else if (warp == 3 && lane == 0) {
      prefetch_tensormap(&thi);
      attn_load_v(sm, &thi, head, seq_start, n_kv, off);
    } else if ((warp == 1 || warp == 2) && lane == 0 && warp - 1 < n_q) {
      attn_mma<kVF16>(sm, tmem, warp - 1, n_kv);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 208;" ::: "memory");
    const int x = (warp - 4) >> 2;
    if (x < n_q)
      attn_softmax<kVF16>(sm, tmem, args, x, n_q, head, seq_start, seq_len, q0 + x * kBM, n_kv, off);
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
  {
    // setmaxnreg.inc only draws on the registers the CTA was launched with:
    // 384 x launch >= 128 x 56 + 256 x 208 needs launch >= 158
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    if (fa.numRegs < kAttnMinLaunchRegs) return cudaErrorInvalidConfiguration;
  }
  AttnArgs a{qkv, cu, out, n_tokens, scale * 1.4426950408889634f};
  dim3 grid((max_seqlen + kBM * kQTiles - 1) / (kBM * kQTiles), 16, n_seqs);
  return launch_pdl(kern, grid, dim3(kThreads), kAttnSmem, st, tlo, thi, a);
}

}  // namespace vitq
