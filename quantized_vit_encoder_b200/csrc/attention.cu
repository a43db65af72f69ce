// Block-diagonal non-causal attention over packed images, head_dim 72, on the
// sm_100a tensor cores.
//
// "Qwen3-VL-8B on RTX 5090", section 3 (FA2 full bidirectional attention per
// ViT block) and section 5 (each image is its own attention window, packed
// with cu_seqlens): O = softmax(Q K^T * scale) V per segment and head.
//
// Design (B200):
//   * one CTA per (segment, head, 256 queries = two 128-row Q tiles); 20 warps:
//     TMA producer, one MMA issuer per Q tile, and eight softmax warps per Q
//     tile, two per TMEM lane quadrant (thread = query row = TMEM lane; each
//     warp of a pair owns 64 of the tile's 128 score columns, and the pair
//     combines its row maxima through shared memory).  S_x(j+1) is computed
//     while the softmax of S_x(j) runs (the softmax frees S_x once it holds it
//     in registers), and the two tiles interleave on the tensor core;
//   * the softmax exponentials run on MUFU ex2; a share can move to a polynomial
//     on the FMA pipe (kPolyEvery).  The softmax warps of tile A and tile B that
//     share an SMSP take turns for their exponentials, so each turn has MUFU to
//     itself while the other tile reads its next scores and waits for its P.V;
//   * K and V are read straight from the packed qkv activation [n, 3, 16, 72]
//     through 3D TMA maps (d, slot, token).  head_dim 72 is padded to 80 by
//     the tensor map itself: d >= 72 lies outside the map so TMA fills zeros,
//     and the padding never exists in HBM.  K: d 0..63 in a 128B-swizzled tile,
//     d 64..79 in a 32B-swizzled tile.  V: d 0..63 and d 64..127 in two
//     128B-swizzled tiles, so that P.V is one N = 80 MMA per 16 keys (two
//     MMAs of N = 64 and 16 cost twice as much: each re-reads P);
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

constexpr int kBM = 128, kBN = 128, kStages = 3, kQTiles = 2;
// Shared memory: a ring of K/V stages, the P tiles (A, B).
constexpr int kKV0 = 0, kKVStride = 53248;
constexpr int kKLo = 0, kKHi = 16384, kVLo = 20480, kVHi = 36864;   // V hi = V lo + 16384 (N-atom stride)
constexpr int kP0 = kKV0 + kStages * kKVStride;         // P tile X: two 64-key atoms of 16 KB
constexpr int kPBytes = 32768;
// Row-maximum exchange of the two softmax warps of a row quadrant:
// [tile][step parity][half][128 rows] fp32 (the last exchange carries the row sums).
constexpr int kRed = kP0 + kQTiles * kPBytes;
constexpr int kBar = kRed + kQTiles * 2 * 2 * 128 * 4;
// barriers: slot 0 (unused), kv_full[S], kv_empty[S], s_full[2], p_full[2], pv_done[2],
// s_free[2], turn[2][4] (the softmax warps of tile x on SMSP q finished their
// exponentials), q_ready[2] (Q tile x is in TMEM), pair[2][4] (both halves of
// tile x, quadrant q, posted their partial row maxima)
constexpr int kNumBars = 1 + 2 * kStages + 4 * kQTiles + kQTiles * 4 + kQTiles + kQTiles * 4;
constexpr size_t kAttnSmem = 1024 + kBar + kNumBars * 8 + 16;
static_assert(kAttnSmem <= 232448, "shared memory budget");
// TMEM columns: S_A 0..127, S_B 128..255, O_A 256..335, Q_A 336..383, O_B 384..463,
// Q_B 464..511 (Q: 40 columns of bf16 pairs, written as 48).
__device__ __forceinline__ uint32_t tmem_s(int x) { return (uint32_t)x * 128u; }
__device__ __forceinline__ uint32_t tmem_o(int x) { return 256u + (uint32_t)x * 128u; }
__device__ __forceinline__ uint32_t tmem_q(int x) { return 336u + (uint32_t)x * 128u; }
// Warpgroup 0: warp 0 TMA producer, warps 1 and 2 MMA issuers for Q tiles A
// and B (warp 3 idle); warps 4-11 softmax of Q tile A, 12-19 of Q tile B (two
// warps per TMEM lane quadrant, each owning 64 of the 128 score columns).
constexpr int kThreads = 128 + 256 * kQTiles;
// Share of the softmax exponentials moved from MUFU to the FMA-pipe polynomial:
// one pair in kPolyEvery (0 = none).  MUFU ex2 runs at 16 per clock per SM.
#ifndef VITQ_ATTN_POLY_EVERY
#define VITQ_ATTN_POLY_EVERY 0
#endif
constexpr int kPolyEvery = VITQ_ATTN_POLY_EVERY;
constexpr int kPolyMod = kPolyEvery > 0 ? kPolyEvery : 1;
// 8-key group of the exponential loop after which the turn passes to the other tile (7 = at the end).
#ifndef VITQ_ATTN_TURN_AT
#define VITQ_ATTN_TURN_AT 5
#endif
constexpr int kTurnAt = VITQ_ATTN_TURN_AT;
// Whether the two tiles' softmax warps of one SMSP take turns for the exponentials.
#ifndef VITQ_ATTN_TURNS
#define VITQ_ATTN_TURNS 1
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
  __device__ uint32_t q_ready(int x) const { return smem_u32(bar(1 + 2 * kStages + 4 * kQTiles + kQTiles * 4 + x)); }
  __device__ uint32_t kv_full(int s) const { return smem_u32(bar(1 + s)); }
  __device__ uint32_t kv_empty(int s) const { return smem_u32(bar(1 + kStages + s)); }
  __device__ uint32_t s_full(int x) const { return smem_u32(bar(1 + 2 * kStages + x)); }
  __device__ uint32_t p_full(int x) const { return smem_u32(bar(1 + 2 * kStages + kQTiles + x)); }
  __device__ uint32_t pv_done(int x) const { return smem_u32(bar(1 + 2 * kStages + 2 * kQTiles + x)); }
  __device__ uint32_t s_free(int x) const { return smem_u32(bar(1 + 2 * kStages + 3 * kQTiles + x)); }
  __device__ uint32_t turn(int x, int q) const { return smem_u32(bar(1 + 2 * kStages + 4 * kQTiles + x * 4 + q)); }
  __device__ uint32_t pair(int x, int q) const {
    return smem_u32(bar(1 + 2 * kStages + 4 * kQTiles + kQTiles * 4 + kQTiles + x * 4 + q));
  }
  __device__ float* red(int x, int par, int h) const {
    return reinterpret_cast<float*>(base + kRed) + ((x * 2 + par) * 2 + h) * 128;
  }
  __device__ uint32_t* tmem_holder() const { return reinterpret_cast<uint32_t*>(bar(kNumBars)); }
  __device__ volatile int* abort_flag() const {
    return reinterpret_cast<volatile int*>(tmem_holder() + 1);
  }
  __device__ uint32_t kv(int s, int part) const { return at(kKV0 + s * kKVStride + part); }
  __device__ uint32_t p(int x) const { return at(kP0 + x * kPBytes); }
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



__device__ void attn_producer(const AttnSmem& sm, const CUtensorMap* tlo, const CUtensorMap* thi,
                              int head, int kv_row0, int n_kv, int off) {
  for (int j = 0; j < n_kv; ++j) {
    const int s = j % kStages;
    const uint32_t ph = (uint32_t)(j / kStages) & 1u;
    if (!mbar_wait(sm.kv_empty(s), ph ^ 1u, sm.abort_flag())) return;
    mbar_arrive_expect_tx(sm.kv_full(s), kKVStride);
    const int row = kv_row0 + kv_tile(j, off, n_kv) * kBN;
    tma_load_3d(sm.kv(s, kKLo), tlo, 0, 16 + head, row, sm.kv_full(s));
    tma_load_3d(sm.kv(s, kKHi), thi, 64, 16 + head, row, sm.kv_full(s));
    tma_load_3d(sm.kv(s, kVLo), tlo, 0, 32 + head, row, sm.kv_full(s));
    tma_load_3d(sm.kv(s, kVHi), tlo, 64, 32 + head, row, sm.kv_full(s));   // d 64..127, >= 72 zero
  }
}

// S_x = Q_x K_j^T (5 MMAs of K = 16 over the padded head_dim 80, Q from TMEM) into S buffer x.
__device__ bool attn_issue_s(const AttnSmem& sm, uint32_t tmem, int x, int j) {
  constexpr uint32_t idesc = make_idesc(1, 1, 0, 0, 128, 128);
  const int s = j % kStages;
  if (!mbar_wait(sm.kv_full(s), (uint32_t)(j / kStages) & 1u, sm.abort_flag())) return false;
  tc_fence_after();
  const uint32_t d = tmem + tmem_s(x), q = tmem + tmem_q(x);
  const uint32_t klo = sm.kv(s, kKLo);
#pragma unroll
  for (int k = 0; k < 4; ++k)
    mma_bf16_ts(d, q + 8 * k, make_smem_desc(klo + 32 * k, 16, 1024, kSwizzle128B), idesc, k > 0 ? 1u : 0u);
  mma_bf16_ts(d, q + 32, make_smem_desc(sm.kv(s, kKHi), 16, 256, kSwizzle32B), idesc, 1u);
  tc_commit(sm.s_full(x));
  return true;
}

// O_x += P_x V_j: P from shared memory (K-major), V MN-major in two 64-wide
// atoms (LBO 16384 bytes apart); one N = 80 MMA per 16 keys.
template <bool kVF16>
__device__ bool attn_issue_pv(const AttnSmem& sm, uint32_t tmem, int x, int j) {
  constexpr uint32_t fmt = kVF16 ? 0u : 1u;
  constexpr uint32_t idesc = make_idesc(fmt, fmt, 0, 1, 128, 80);
  if (!mbar_wait(sm.p_full(x), (uint32_t)j & 1u, sm.abort_flag())) return false;
  VITQ_TRACE_EV(14 + x, j);   // mma: P complete
  tc_fence_after();
  const int s = j % kStages;
  const uint32_t vlo = sm.kv(s, kVLo), p0 = sm.p(x);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint64_t ad = make_smem_desc(p0 + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024, kSwizzle128B);
    const uint32_t acc = (j > 0 || k > 0) ? 1u : 0u;
    mma_bf16_ss(tmem + tmem_o(x), ad, make_smem_desc(vlo + k * 2048, kVHi - kVLo, 1024, kSwizzle128B), idesc, acc);
  }
  tc_commit(sm.pv_done(x));
  return true;
}

// Tensor-core work of Q tile x, issued by its own thread.  S_x(j+1) is issued as
// soon as the softmax has moved S_x(j) into registers (s_free), so it overlaps
// that softmax; P_x(j).V_j follows when P_x(j) is in shared memory.  The two
// tiles' threads interleave on the tensor core; a K/V stage is released when
// both tiles' P.V of that stage have completed (kv_empty counts one commit per tile).
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
    tc_commit(sm.kv_empty(j % kStages));
  }
}

__device__ __forceinline__ uint32_t pack_p(float lo, float hi, bool f16) {
  if (f16) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  return pack_bf16x2(lo, hi);
}

// Two warps per (Q tile, TMEM lane quadrant); thread = query row = TMEM lane.
// Half h of the pair owns score columns 64h..64h+63 of its rows and P atom h.
// The halves combine their row maxima through shared memory every step (so
// both follow the same running max); the row sums stay partial until the end.
// Half 0 also copies the Q rows into TMEM, rescales O and writes the output.
template <bool kVF16>
__device__ void attn_softmax(const AttnSmem& sm, uint32_t tmem, const AttnArgs& g, int x, int h, int n_q,
                             int head, int seq_start, int seq_len, int q0, int n_kv, int off) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quad = warp & 3;
  const int r = quad * 32 + lane;
  const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
  const uint32_t s_addr = tmem + lane_addr + tmem_s(x) + 64 * h, o_addr = tmem + lane_addr + tmem_o(x);
  uint8_t* pbase = sm.base + kP0 + x * kPBytes + h * 16384;
  const bool tr = h == 0 && quad == 0 && lane == 0;
  (void)tr;
  if (h == 0) {
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
    // keys of this tile inside the segment, counted from this half's first column
    const int valid = seq_len - kv_tile(j, off, n_kv) * kBN - 64 * h;
    uint32_t su[2][32];
    tmem_ld32(s_addr, su[0]);
    tmem_ld32(s_addr + 32, su[1]);
    tmem_wait_ld();
    if (tr) VITQ_TRACE_EV(26 + x, j);   // softmax: S in registers
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(sm.s_free(x));
    if (valid < 64) {
#pragma unroll
      for (int i = 0; i < 64; ++i)
        if (i >= valid) su[i >> 5][i & 31] = 0xFF800000u;   // -inf
    }
    // partial row max: 8 independent chains of 3-input max, then a tree
    float mp[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) mp[k] = __uint_as_float(su[0][k]);
#pragma unroll
    for (int i = 8; i < 64; i += 16)
#pragma unroll
      for (int k = 0; k < 8; ++k)
        mp[k] = fmax3(mp[k], __uint_as_float(su[(i + k) >> 5][(i + k) & 31]),
                      __uint_as_float(su[(i + 8 + k) >> 5][(i + 8 + k) & 31]));
    const float pm = fmax3(fmax3(mp[0], mp[1], mp[2]), fmax3(mp[3], mp[4], mp[5]), fmaxf(mp[6], mp[7]));
    sm.red(x, j & 1, h)[r] = pm;
    __syncwarp();
    if (lane == 0) mbar_arrive(sm.pair(x, quad));
    ok = mbar_wait(sm.pair(x, quad), (uint32_t)j & 1u, sm.abort_flag());
    if (!__all_sync(0xffffffffu, ok)) return;
    const float mx = fmaxf(pm, sm.red(x, j & 1, 1 - h)[r]) * g.scale_log2;
    if (j > 0) {
      // P(j) overwrites P(j-1), and half 0 may rescale O: P(j-1).V must be done
      ok = mbar_wait(sm.pv_done(x), (uint32_t)(j - 1) & 1u, sm.abort_flag());
      if (!__all_sync(0xffffffffu, ok)) return;
      tc_fence_after();
    }
    if (tr) VITQ_TRACE_EV(22 + x, j);   // softmax: max known, O stable
    // new running max: it changes only when the tile max exceeds it by more than 8
    // (so P <= 2^8), and the decision is warp-uniform because the O rescale uses
    // warp-collective tcgen05.ld/st (rows that keep their max get alpha = 1).
    // Both halves see the same maxima, so they take the same decisions.
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
    // P = 2^(s * scale_log2 - m_run), rounded to the P.V operand type, into this
    // half's 64-key atom of the swizzled P tile; 8 fp32 partial row sums.
    const uint64_t sc2 = f2pack(g.scale_log2, g.scale_log2), nm2 = f2pack(-m_run, -m_run);
    uint64_t ls[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int k0 = c * 8 + 2 * i;
        const float2 t = f2unpack(ffma2(f2pack(__uint_as_float(su[k0 >> 5][k0 & 31]),
                                               __uint_as_float(su[(k0 + 1) >> 5][(k0 + 1) & 31])),
                                        sc2, nm2));
        // every kPolyEvery-th pair runs the FMA-pipe polynomial, the rest MUFU ex2
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
      uint8_t* dst = pbase + r * 128 + ((c ^ (r & 7)) << 4);
      *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
      // hand the turn to the other tile a little before the end, so that its
      // exponentials start while these finish (hides the hand-over latency)
      if (kTakeTurns && c == kTurnAt && n_q == 2 && !(x == 1 && j == n_kv - 1)) {
        __syncwarp();
        if (lane == 0) mbar_arrive(sm.turn(x, quad));
      }
    }
    if (rescale && h == 0) {
      // O (complete up to P.V(j-1)) to the new max; done after P so the scores are dead
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
    if (lane == 0) mbar_arrive(sm.p_full(x));
  }
  bool ok = mbar_wait(sm.pv_done(x), (uint32_t)(n_kv - 1) & 1u, sm.abort_flag());
  if (!__all_sync(0xffffffffu, ok)) return;
  tc_fence_after();
  // row sum = the two halves' partial sums (one more exchange, slot parity n_kv)
  sm.red(x, n_kv & 1, h)[r] = l_run;
  __syncwarp();
  if (lane == 0) mbar_arrive(sm.pair(x, quad));
  ok = mbar_wait(sm.pair(x, quad), (uint32_t)n_kv & 1u, sm.abort_flag());
  if (!__all_sync(0xffffffffu, ok)) return;
  if (h != 0) return;
  const float l_sum = l_run + sm.red(x, n_kv & 1, 1)[r];
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
    for (int s = 0; s < kStages; ++s) {
      mbar_init(sm.kv_full(s), 1);
      mbar_init(sm.kv_empty(s), (uint32_t)n_q);       // one commit per active Q tile
    }
    for (int x = 0; x < kQTiles; ++x) {
      for (int q = 0; q < 4; ++q) mbar_init(sm.turn(x, q), 2);
      for (int q = 0; q < 4; ++q) mbar_init(sm.pair(x, q), 2);
      mbar_init(sm.q_ready(x), 4);
      mbar_init(sm.s_full(x), 1);
      mbar_init(sm.p_full(x), 8);
      mbar_init(sm.pv_done(x), 1);
      mbar_init(sm.s_free(x), 8);
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
    if (warp == 0 && lane == 0) {
      prefetch_tensormap(&tlo);
      prefetch_tensormap(&thi);
      attn_producer(sm, &tlo, &thi, head, seq_start, n_kv, off);
    } else if ((warp == 1 || warp == 2) && lane == 0 && warp - 1 < n_q) {
      attn_mma<kVF16>(sm, tmem, warp - 1, n_kv);
    }
  } else {
    const int x = (warp - 4) >> 3, h = ((warp - 4) >> 2) & 1;
    if (x < n_q)
      attn_softmax<kVF16>(sm, tmem, args, x, h, n_q, head, seq_start, seq_len, q0 + x * kBM, n_kv, off);
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
  AttnArgs a{qkv, cu, out, n_tokens, scale * 1.4426950408889634f};
  dim3 grid((max_seqlen + kBM * kQTiles - 1) / (kBM * kQTiles), 16, n_seqs);
  return launch_pdl(kern, grid, dim3(kThreads), kAttnSmem, st, tlo, thi, a);
}

}  // namespace vitq
