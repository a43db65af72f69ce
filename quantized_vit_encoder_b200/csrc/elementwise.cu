// Memory-bound kernels of the ViT block: FP8 block-128 activation quantisation
// (standalone, fused after LayerNorm, fused after GELU), 128x128 weight
// quantisation, the 2D rotary table and its in-place application, and the
// per-patch (row, col) positions of packed images.
//
// Quantisation convention ("Qwen3-VL-8B on RTX 5090", section 3, fused
// per-token / per-128-K-block FP8 activation quant; scale = amax / 448 as in
// "qwen3_omni: record why FP8 is not shipped", recipe): for each row and each
// group of 128 columns, s = amax / 448 (IEEE fp32 division) and
// code = E4M3_RNE_satfinite(y / s) (IEEE fp32 division).  A zero scale gives
// zero codes.  Scales are stored kb-major: s[kb * lds + row].
#include "internal.h"
#include "ptx.cuh"

#include <cuda_fp16.h>

namespace vitq {

namespace {

constexpr float kE4M3Max = 448.0f;

// Two fp32 values (packed) -> bf16x2, round to nearest even (lo in bits 0..15).
__device__ __forceinline__ uint32_t bf16x2_of(uint64_t v) {
  const float2 f = f2unpack(v);
  uint32_t w;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w) : "f"(f.y), "f"(f.x));
  return w;
}
// ------------------------------------------------ exact block-128 quantisation
// Group scale fl32(amax / 448) without a division: q0 = fl(amax * R) with
// R = fl(1/448), then one FMA correction.  For every bf16 amax from 2^-100 to
// the largest finite bf16 this equals the IEEE quotient (each of them checked
// on the host in exact rational arithmetic); every amax here is a bf16 value
// (the quantised inputs are bf16).  Other values take the IEEE division.
__device__ __forceinline__ float e4m3_scale(float amax) {
  if (amax >= 7.88860905e-31f && amax <= 3.38953139e38f) {
    constexpr float R = 1.0f / 448.0f;
    const float q0 = __fmul_rn(amax, R);
    return __fmaf_rn(__fmaf_rn(-q0, kE4M3Max, amax), R, q0);
  }
  return __fdiv_rn(amax, kE4M3Max);
}

// Four fp32 values -> four E4M3 codes in one word (round to nearest even,
// saturate to +-448), value i in byte i.
__device__ __forceinline__ uint32_t cvt4_e4m3(float a0, float a1, float a2, float a3) {
  uint32_t w;
  asm("{.reg .b16 l, h; cvt.rn.satfinite.e4m3x2.f32 l, %2, %1; cvt.rn.satfinite.e4m3x2.f32 h, %4, %3;"
      " mov.b32 %0, {l, h};}"
      : "=r"(w) : "f"(a0), "f"(a1), "f"(a2), "f"(a3));
  return w;
}

// E4M3 codes of fl32(v_i / s) by IEEE division (the rare cases of quant8).
__device__ __noinline__ uint2 quant8_divide(float v0, float v1, float v2, float v3, float v4, float v5, float v6,
                                            float v7, float s) {
  return make_uint2(cvt4_e4m3(__fdiv_rn(v0, s), __fdiv_rn(v1, s), __fdiv_rn(v2, s), __fdiv_rn(v3, s)),
                    cvt4_e4m3(__fdiv_rn(v4, s), __fdiv_rn(v5, s), __fdiv_rn(v6, s), __fdiv_rn(v7, s)));
}

// E4M3 codes of 8 values of one group, equal to code(fl32(y / s)) without a
// division.  r = rcp.approx(s) is within 1 ulp of 1/s, so rl = r - 64 ulps
// <= 1/s <= r + 64 ulps = rh.  For y >= 0, y rl <= y / s <= y rh, and rounding
// to fp32 and then to E4M3 is monotone, so code(fl(y rl)) <= code(fl(y / s))
// <= code(fl(y rh)) (mirrored for y < 0): where the outer codes agree, they are
// the answer.  A group where they differ (about 2^-10 of groups) divides
// exactly.  A scale below the fp32 normal range (amax < 448 * 2^-126), or an
// infinite or NaN one, divides exactly; a zero scale gives zero codes.
__device__ __forceinline__ uint2 quant8(const float (&v)[8], float s) {
  if (s >= 1.17549435e-38f && s <= 1e36f) {   // normal, with a normal reciprocal
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(s));
    const uint32_t rb = __float_as_uint(r);
    const uint64_t rl = f2pack(__uint_as_float(rb - 64u), __uint_as_float(rb - 64u));
    const uint64_t rh = f2pack(__uint_as_float(rb + 64u), __uint_as_float(rb + 64u));
    float a[8], b[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint64_t x = f2pack(v[2 * i], v[2 * i + 1]);
      const float2 p = f2unpack(fmul2(x, rl)), q = f2unpack(fmul2(x, rh));
      a[2 * i] = p.x;
      a[2 * i + 1] = p.y;
      b[2 * i] = q.x;
      b[2 * i + 1] = q.y;
    }
    uint2 w = make_uint2(cvt4_e4m3(a[0], a[1], a[2], a[3]), cvt4_e4m3(a[4], a[5], a[6], a[7]));
    const uint32_t h0 = cvt4_e4m3(b[0], b[1], b[2], b[3]), h1 = cvt4_e4m3(b[4], b[5], b[6], b[7]);
    if ((w.x != h0) | (w.y != h1))   // rare: a value straddles an E4M3 rounding boundary
      w = quant8_divide(v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7], s);
    return w;
  }
  if (s != 0.f) return quant8_divide(v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7], s);
  return make_uint2(0u, 0u);
}

// Max of |x| over 8 bf16 values (one uint4), as a bf16 bit pattern: the
// magnitudes of bf16 values order like their bit patterns with the sign
// cleared, so a packed 16-bit integer max finds it.  A NaN input wins (and
// makes the group's scale NaN, as the IEEE definition of the max does).
__device__ __forceinline__ uint32_t amax_bits8(const uint4& u) {
  uint32_t m;
  asm("{.reg .b32 t0, t1; max.u16x2 t0, %1, %2; max.u16x2 t1, %3, %4; max.u16x2 %0, t0, t1;}"
      : "=r"(m)
      : "r"(u.x & 0x7FFF7FFFu), "r"(u.y & 0x7FFF7FFFu), "r"(u.z & 0x7FFF7FFFu), "r"(u.w & 0x7FFF7FFFu));
  return max(m & 0xFFFFu, m >> 16);
}

// Max over each half warp of bf16 bit patterns, as a float: lanes 0-15 get the
// max of lanes 0-15, lanes 16-31 that of lanes 16-31.  All 32 lanes must take part.
__device__ __forceinline__ float half_warp_max_bits(uint32_t m, int lane) {
  const uint32_t m0 = __reduce_max_sync(0xffffffffu, lane < 16 ? m : 0u);
  const uint32_t m1 = __reduce_max_sync(0xffffffffu, lane < 16 ? 0u : m);
  return __uint_as_float((lane < 16 ? m0 : m1) << 16);
}

__device__ __forceinline__ void unpack8(const uint4& u, float (&v)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ void load8_bf16(const __nv_bfloat16* p, float (&v)[8]) {
  unpack8(*reinterpret_cast<const uint4*>(p), v);
}

// Lane layout shared by the row kernels: a warp covers 256 columns per step;
// lanes 0-15 hold group 2*step, lanes 16-31 group 2*step+1, 8 columns each.
__device__ __forceinline__ int lane_col(int step, int lane) { return step * 256 + lane * 8; }

// Group amax over the half warp, scale, codes and scale store for one step
// (lane layout of lane_col; all 32 lanes take part).  raw: the lane's 8 bf16
// values (zeros past K).
__device__ __forceinline__ void quant_store(const uint4& raw, bool ok, int lane, int row, int col, int K,
                                            uint8_t* __restrict__ q, float* __restrict__ s, int lds) {
  const float sc = e4m3_scale(half_warp_max_bits(amax_bits8(raw), lane));
  if (ok) {
    float v[8];
    unpack8(raw, v);
    *reinterpret_cast<uint2*>(q + (size_t)row * K + col) = quant8(v, sc);
    if ((lane & 15) == 0) s[(size_t)(col >> 7) * lds + row] = sc;
  }
}

// ------------------------------------------------------------ activation quant
// One warp per row; every load of the row is issued before any use.

template <int ITERS>
__global__ void __launch_bounds__(128, 12) quant_act_kernel(const __nv_bfloat16* __restrict__ x, int M, int K, int ldx,
                                 uint8_t* __restrict__ q, float* __restrict__ s, int lds) {
  pdl_trigger();
  pdl_wait();
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  uint4 raw[ITERS];
#pragma unroll
  for (int it = 0; it < ITERS; ++it) {
    const int col = lane_col(it, lane);
    raw[it] = col < K ? *reinterpret_cast<const uint4*>(x + (size_t)row * ldx + col) : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int it = 0; it < ITERS; ++it) {
    const int col = lane_col(it, lane);
    quant_store(raw[it], col < K, lane, row, col, K, q, s, lds);
  }
}

// --------------------------------------------------------- LayerNorm + quant
// "Qwen3-VL-8B on RTX 5090", section 3: LayerNorm with the FP8 quantisation of
// its bf16 output fused in (the normalised activation never goes to HBM).
// A half warp per row (lane l of the half holds columns 128c + 8l, so each
// 128-column group is one chunk c across the half warp), eight rows per CTA;
// gamma, beta and the bracket term below are staged once per CTA in shared
// memory as fp32.  The statistics are exact fp64 sums of the bf16 inputs (sum
// and sum of squares).  The normalised value y = (x - mean) rstd gamma + beta
// is evaluated in fp32; its error is below e = (|y| + 2|beta|) 2^-20 + 2^-126,
// and where y - e and y + e round to the same bf16 value, that value is the
// rounding of the exact y.  Elsewhere (about 2^-11 of the pairs) y is
// recomputed in fp64.

// bf16 pair of ((x - mean) rstd gamma + beta) evaluated in fp64.
__device__ __noinline__ uint32_t ln_pair_fp64(float x0, float x1, float g0, float g1, float b0, float b1,
                                              double mean, double rstd) {
  const __nv_bfloat16 h0 = __double2bfloat16(((double)x0 - mean) * rstd * (double)g0 + (double)b0);
  const __nv_bfloat16 h1 = __double2bfloat16(((double)x1 - mean) * rstd * (double)g1 + (double)b1);
  return (uint32_t)*reinterpret_cast<const uint16_t*>(&h0) | ((uint32_t)*reinterpret_cast<const uint16_t*>(&h1) << 16);
}

constexpr int kLnRows = 8;

constexpr int kLnMaxChunks = 36;   // K <= 4608

// ITERS = chunks per row (1..9, unrolled), or 0: wider rows, chunk count from K.
template <int ITERS, bool kOutBf16>
__global__ void __launch_bounds__(16 * kLnRows, 6)
    ln_quant_kernel(const __nv_bfloat16* __restrict__ x, int ldx, const __nv_bfloat16* __restrict__ gamma,
                    const __nv_bfloat16* __restrict__ beta, int M, int K, double eps,
                    uint8_t* __restrict__ q, float* __restrict__ s, int lds, __nv_bfloat16* __restrict__ y) {
  // per column: gamma, beta, (2|beta| 2^-20 + 2^-126), as fp32 (dynamic shared memory,
  // nch * 1536 bytes).  Columns 128c + 8l + 4h .. +3 sit in float4 (2c + h) * 16 + l, so
  // the 16 lanes of a half warp read 16 consecutive float4.
  extern __shared__ float4 ln_smem[];
  const int nch = ITERS > 0 ? ITERS : (K + 127) >> 7;
  float4* sg = ln_smem;
  float4* sb = ln_smem + nch * 32;
  float4* se = ln_smem + 2 * nch * 32;
  pdl_trigger();
  for (int i = threadIdx.x; i < nch * 16; i += blockDim.x) {
    const int col = i * 8;
    float g[8], b[8];
    if (col < K) {
      load8_bf16(gamma + col, g);
      load8_bf16(beta + col, b);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) g[k] = b[k] = 0.f;
    }
    const int j0 = ((i >> 4) * 2) * 16 + (i & 15), j1 = j0 + 16;
    sg[j0] = make_float4(g[0], g[1], g[2], g[3]);
    sg[j1] = make_float4(g[4], g[5], g[6], g[7]);
    sb[j0] = make_float4(b[0], b[1], b[2], b[3]);
    sb[j1] = make_float4(b[4], b[5], b[6], b[7]);
    float e[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) e[k] = fmaf(fabsf(b[k]), 0x1p-19f, 0x1p-126f);
    se[j0] = make_float4(e[0], e[1], e[2], e[3]);
    se[j1] = make_float4(e[4], e[5], e[6], e[7]);
  }
  __syncthreads();
  pdl_wait();   // x may be the previous kernel's output
  const int lane = threadIdx.x & 31, l = lane & 15;
  const int row = blockIdx.x * kLnRows + (threadIdx.x >> 4);
  // both halves of a warp stay to the end (the group max is a full-warp reduction)
  if (blockIdx.x * kLnRows + ((threadIdx.x >> 5) << 1) >= M) return;
  const bool row_ok = row < M;
  const __nv_bfloat16* xr = x + (size_t)(row_ok ? row : 0) * ldx;
  // the second pass reads the row again (from L1, where the first pass left it)
  auto load_chunk = [&](int c) {
    const int col = c * 128 + l * 8;
    return (row_ok && col < K) ? *reinterpret_cast<const uint4*>(xr + col) : make_uint4(0, 0, 0, 0);
  };
  // exact fp64 sums of the bf16 inputs (bf16 -> fp32 -> fp64 is exact); 2 chains each
  double s1[2] = {0.0, 0.0}, s2[2] = {0.0, 0.0};
#pragma unroll
  for (int c = 0; c < nch; ++c) {
    float v[8];
    unpack8(load_chunk(c), v);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const double d = (double)v[i];
      s1[i & 1] += d;
      s2[i & 1] = fma(d, d, s2[i & 1]);
    }
  }
  double t1 = s1[0] + s1[1], t2 = s2[0] + s2[1];
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) {
    t1 += __shfl_xor_sync(0xffffffffu, t1, o);
    t2 += __shfl_xor_sync(0xffffffffu, t2, o);
  }
  const double mean = t1 / (double)K;
  const double var = fmax(t2 / (double)K - mean * mean, 0.0);
  const double rstd = 1.0 / sqrt(var + eps);
  const float mh = (float)mean, ml = (float)(mean - (double)mh), r32 = (float)rstd;
  const uint64_t nmh = f2pack(-mh, -mh), nml = f2pack(-ml, -ml), rr = f2pack(r32, r32);
#pragma unroll
  for (int c = 0; c < nch; ++c) {
    const int col = c * 128 + l * 8;
    const bool ok = row_ok && col < K;
    float v[8];
    unpack8(load_chunk(c), v);
    const int j0 = c * 32 + l, j1 = j0 + 16;
    const float4 g0 = sg[j0], g1 = sg[j1], b0 = sb[j0], b1 = sb[j1], e0 = se[j0], e1 = se[j1];
    const float g[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
    const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
    const float eb[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
    uint4 wq;
    uint32_t* w = reinterpret_cast<uint32_t*>(&wq);
    uint32_t slow = 0u;   // pairs whose bracket straddles a bf16 rounding boundary
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint64_t t = fmul2(fadd2(fadd2(f2pack(v[2 * i], v[2 * i + 1]), nmh), nml), rr);
      const uint64_t yy = ffma2(t, f2pack(g[2 * i], g[2 * i + 1]), f2pack(b[2 * i], b[2 * i + 1]));
      const float2 yf = f2unpack(yy);
      const uint64_t e = ffma2(f2pack(fabsf(yf.x), fabsf(yf.y)), f2pack(0x1p-20f, 0x1p-20f),
                               f2pack(eb[2 * i], eb[2 * i + 1]));
      const uint32_t lo = bf16x2_of(ffma2(e, f2pack(-1.f, -1.f), yy)), hi = bf16x2_of(fadd2(yy, e));
      slow |= (uint32_t)(lo != hi) << i;
      w[i] = lo;
    }
    if (slow) {   // rare (about 2^-11 of the pairs): those pairs in fp64 (unrolled: a
                  // runtime index would put v, g, b and w in local memory for every chunk)
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if ((slow >> i) & 1u)
          w[i] = ln_pair_fp64(v[2 * i], v[2 * i + 1], g[2 * i], g[2 * i + 1], b[2 * i], b[2 * i + 1], mean, rstd);
    }
    if (kOutBf16) {   // bf16 output (the bf16 blocks and mergers)
      if (ok) *reinterpret_cast<uint4*>(y + (size_t)row * K + col) = wq;
    } else {
      const float sc = e4m3_scale(half_warp_max_bits(amax_bits8(wq), lane));
      if (ok) {
        float o[8];
        unpack8(wq, o);
        *reinterpret_cast<uint2*>(q + (size_t)row * K + col) = quant8(o, sc);
        if (l == 0) s[(size_t)c * lds + row] = sc;
      }
    }
  }
}

// ------------------------------------------------------------- GELU + quant
// "Qwen3-VL-8B on RTX 5090", section 3: GELU(tanh) on the fc1 output with the FP8
// quantisation for fc2 fused in.
// GELU(tanh) = 0.5 x (1 + tanh(u)) = x / (1 + exp(-2u)), u = sqrt(2/pi)(x + 0.044715 x^3).
// Its input is a bf16 value (the rounded fc1 output), so the bf16 result is a
// function of 16 bits: g_gelu_table holds it for every bf16 bit pattern,
// evaluated once per device in fp64 (the sigmoid form does not cancel for
// u << 0) and rounded to bf16.  The GELU pass is then one shared-memory lookup
// per element followed by the block-128 quantisation.

__device__ uint16_t g_gelu_table[65536];

__global__ void gelu_table_kernel() {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= 65536) return;
  const float x = __uint_as_float((uint32_t)i << 16);
  const double xd = (double)x;
  const double ud = 0.79788456080286535588 * (xd + 0.044715 * xd * xd * xd);
  const __nv_bfloat16 g = __double2bfloat16(xd / (1.0 + exp(-2.0 * ud)));
  g_gelu_table[i] = *reinterpret_cast<const uint16_t*>(&g);
}

constexpr int kGeluThreads = 1024;
constexpr size_t kGeluSmem = 65536 * 2;

// Persistent: one CTA per SM copies the table into shared memory, then each warp
// takes (row, 256-column step) items w, w + W, w + 2W, ... (W = warps in the
// grid; lane layout of lane_col), stepping (row, step) incrementally.  The next
// item's 8 inputs per lane are loaded before the current item is processed, so
// the load latency overlaps the work.
__global__ void __launch_bounds__(kGeluThreads, 1)
    gelu_quant_kernel(const __nv_bfloat16* f, int M, int K, int ldf, uint8_t* __restrict__ q,
                      float* __restrict__ s, int lds, __nv_bfloat16* y) {
  extern __shared__ __align__(16) uint16_t lut[];
  pdl_trigger();
  {
    const uint4* src = reinterpret_cast<const uint4*>(g_gelu_table);
    uint4* dst = reinterpret_cast<uint4*>(lut);
#pragma unroll
    for (int i = 0; i < 8; ++i) dst[threadIdx.x + i * kGeluThreads] = src[threadIdx.x + i * kGeluThreads];
  }
  __syncthreads();
  pdl_wait();
  const int steps = (K + 255) / 256;
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * (kGeluThreads / 32);
  const int w0 = blockIdx.x * (kGeluThreads / 32) + (threadIdx.x >> 5);
  const int drow = warps / steps, dst_ = warps - drow * steps;   // item stride as (rows, steps)
  int row = w0 / steps, st = w0 - row * steps;
  auto load = [&](int r, int t) {
    const int col = lane_col(t, lane);
    return (r < M && col < K) ? *reinterpret_cast<const uint4*>(f + (size_t)r * ldf + col) : make_uint4(0u, 0u, 0u, 0u);
  };
  uint4 cur = load(row, st);
  while (row < M) {
    int nrow = row + drow, nst = st + dst_;
    if (nst >= steps) {
      nst -= steps;
      ++nrow;
    }
    const uint4 nxt = load(nrow, nst);
    const int col = lane_col(st, lane);
    const bool ok = col < K;
    const uint32_t wd[4] = {cur.x, cur.y, cur.z, cur.w};
    uint4 g;
    uint32_t* gv = reinterpret_cast<uint32_t*>(&g);
#pragma unroll
    for (int i = 0; i < 4; ++i)   // zero inputs (past K) read GELU(0) = 0
      gv[i] = (uint32_t)lut[wd[i] & 0xFFFFu] | ((uint32_t)lut[wd[i] >> 16] << 16);
    if (y) {   // bf16 output (may be f itself: each lane reads its 8 values before writing them)
      if (ok) *reinterpret_cast<uint4*>(y + (size_t)row * ldf + col) = g;
    } else {
      quant_store(g, ok, lane, row, col, K, q, s, lds);
    }
    cur = nxt;
    row = nrow;
    st = nst;
  }
}

// ------------------------------------------------------------ weight quant
// One CTA (256 threads) per 128x128 block of W [N, K].

__global__ void quant_weight_kernel(const __nv_bfloat16* __restrict__ w, int N, int K,
                                    uint8_t* __restrict__ q, float* __restrict__ s) {
  pdl_trigger();
  pdl_wait();
  const int nb = blockIdx.y, kb = blockIdx.x;
  const int nkb = gridDim.x;
  const int t = threadIdx.x;
  // 128 rows x 16 chunks of 8 columns = 2048 chunks, 8 per thread.
  float a = 0.f;
  for (int c = t; c < 2048; c += 256) {
    const int r = nb * 128 + (c >> 4);
    const int col = kb * 128 + (c & 15) * 8;
    if (r < N && col < K) {
      float v[8];
      load8_bf16(w + (size_t)r * K + col, v);
#pragma unroll
      for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(v[i]));
    }
  }
  __shared__ float red[8];
  a = warp_max(a);
  if ((t & 31) == 0) red[t >> 5] = a;
  __syncthreads();
  if (t < 32) {
    float b = t < 8 ? red[t] : 0.f;
    b = warp_max(b);
    if (t == 0) red[0] = b;
  }
  __syncthreads();
  const float sc = __fdiv_rn(red[0], kE4M3Max);
  if (t == 0) s[nb * nkb + kb] = sc;
  for (int c = t; c < 2048; c += 256) {
    const int r = nb * 128 + (c >> 4);
    const int col = kb * 128 + (c & 15) * 8;
    if (r < N && col < K) {
      float v[8];
      load8_bf16(w + (size_t)r * K + col, v);
      *reinterpret_cast<uint2*>(q + (size_t)r * K + col) = quant8(v, sc);
    }
  }
}

// --------------------------------------------------------------- 2D rotary
// "Qwen3-VL-8B on RTX 5090", section 3 (2D rotate_half rotary after the QKV
// projection) and "spark_model/layers/vision_encoder.rs" (rope_inv_freq: head_dim/4
// = 18 frequencies, used for the row and for the column).
// Table layout: cos_sin[t * 72 + j] = cos(angle_j), cos_sin[t * 72 + 36 + j] = sin(angle_j),
// angle_j = row * f_j (j < 18), col * f_(j-18) (18 <= j < 36), f_i = theta^(-2i/36).

__global__ void rope_table_kernel(const int32_t* __restrict__ pos, int n, double theta,
                                  float* __restrict__ cs) {
  pdl_trigger();
  pdl_wait();
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n * 36) return;
  const int t = idx / 36, j = idx - t * 36;
  const int i = j < 18 ? j : j - 18;
  const double f = pow(theta, -2.0 * (double)i / 36.0);
  const double p = (double)pos[2 * t + (j < 18 ? 0 : 1)];
  double sn, cn;
  sincos(p * f, &sn, &cn);
  cs[(size_t)t * 72 + j] = (float)cn;
  cs[(size_t)t * 72 + 36 + j] = (float)sn;
}

// One thread per work item, 432 items per token, no barrier: items 0..287 are
// (q/k head slot, group of four rotary pairs): the thread reads x_j .. x_(j+3)
// and their partners x_(j+36) .. x_(j+39) (8 bytes each) and writes both,
// x'_j = x_j c_j - x_(j+36) s_j and x'_(j+36) = x_(j+36) c_j + x_j s_j, so no
// thread reads what another writes.  Items 288..431 are the 8-element chunks of
// the v heads, converted to fp16 in place when v_to_f16 (round to nearest:
// exact for 2^-14 <= |v| <= 65504, within 2^-25 below; larger |v| is clamped to
// 65504 and flagged in the device error word).
constexpr int kRopeItems = 432;

__global__ void __launch_bounds__(256) rope_apply_kernel(__nv_bfloat16* __restrict__ qkv,
                                                         const float* __restrict__ cs, int n, int v_to_f16) {
  pdl_trigger();
  pdl_wait();
  const long long g = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int t = (int)(g / kRopeItems), w = (int)(g - (long long)t * kRopeItems);
  if (t >= n) return;
  __nv_bfloat16* base = qkv + (size_t)t * 3456;
  if (w < 288) {
    const int slot = w / 9, p = w - slot * 9, j = 4 * p;
    uint2* lo = reinterpret_cast<uint2*>(base + slot * 72 + j);
    uint2* hi = reinterpret_cast<uint2*>(base + slot * 72 + 36 + j);
    const uint2 a = *lo, b = *hi;
    const float4 c = __ldg(reinterpret_cast<const float4*>(cs + (size_t)t * 72 + j));
    const float4 sn = __ldg(reinterpret_cast<const float4*>(cs + (size_t)t * 72 + 36 + j));
    const float2 a0 = unpack_bf16x2(a.x), a1 = unpack_bf16x2(a.y), b0 = unpack_bf16x2(b.x), b1 = unpack_bf16x2(b.y);
    const float x[4] = {a0.x, a0.y, a1.x, a1.y}, y[4] = {b0.x, b0.y, b1.x, b1.y};
    const float cv[4] = {c.x, c.y, c.z, c.w}, sv[4] = {sn.x, sn.y, sn.z, sn.w};
    float xo[4], yo[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      xo[i] = fmaf(x[i], cv[i], -y[i] * sv[i]);
      yo[i] = fmaf(y[i], cv[i], x[i] * sv[i]);
    }
    *lo = make_uint2(pack_bf16x2(xo[0], xo[1]), pack_bf16x2(xo[2], xo[3]));
    *hi = make_uint2(pack_bf16x2(yo[0], yo[1]), pack_bf16x2(yo[2], yo[3]));
  } else if (v_to_f16) {
    __nv_bfloat16* dst = base + 2304 + (w - 288) * 8;
    float v[8];
    load8_bf16(dst, v);
    // fp16 holds |v| <= 65504: larger values are clamped to +-65504 and raise the
    // range bit of the device error word (NaN passes through unchanged)
    bool big = false;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (fabsf(v[i]) > 65504.f) {
        v[i] = copysignf(65504.f, v[i]);
        big = true;
      }
    }
    if (big) atomicOr(&g_device_error, kErrValueRange);
    __half2 h0 = __floats2half2_rn(v[0], v[1]), h1 = __floats2half2_rn(v[2], v[3]);
    __half2 h2 = __floats2half2_rn(v[4], v[5]), h3 = __floats2half2_rn(v[6], v[7]);
    *reinterpret_cast<uint4*>(dst) = make_uint4(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1),
                                                *reinterpret_cast<uint32_t*>(&h2), *reinterpret_cast<uint32_t*>(&h3));
  }
}

// --------------------------------------------------------------- positions
// Token order inside an h x w image: 2x2-block order for even grids (block
// (br, bc) row-major, inside it (0,0) (0,1) (1,0) (1,1)), row-major otherwise.

// Image of token t of the packed images, and the token's (row, col) in that image:
// 2x2-block order (merger neighbours consecutive) for even grids, row-major otherwise.
__device__ __forceinline__ void token_place(const GridList& grids, int t, int& img, int& r, int& c) {
  int start = 0;
  for (img = 0; img < grids.n - 1; ++img) {
    const int len = grids.hw[2 * img] * grids.hw[2 * img + 1];
    if (t < start + len) break;
    start += len;
  }
  const int h = grids.hw[2 * img], w = grids.hw[2 * img + 1];
  const int p = t - start;
  if ((h & 1) == 0 && (w & 1) == 0) {
    const int blk = p >> 2, within = p & 3;
    const int br = blk / (w >> 1), bc = blk - br * (w >> 1);
    r = 2 * br + (within >> 1);
    c = 2 * bc + (within & 1);
  } else {
    r = p / w;
    c = p - r * w;
  }
}

// ------------------------------------------------- interpolated position embedding
// "Qwen3-VL-8B on RTX 5090", section 3 (patch_embed -> + interpolated pos_embed):
// the learned 48 x 48 table is interpolated bilinearly to each image's patch grid,
// sample points running corner to corner (row r of h at r * 47 / (h - 1)).  fp64
// weights and sums of the bf16 table values, rounded once to bf16.  One CTA of 144
// threads per token, 8 channels per thread.
constexpr int kPosGrid = 48;

__global__ void __launch_bounds__(144) pos_interp_kernel(GridList grids, const __nv_bfloat16* __restrict__ table,
                                                         __nv_bfloat16* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  const int t = blockIdx.x;
  int img, r, c;
  token_place(grids, t, img, r, c);
  const int h = grids.hw[2 * img], w = grids.hw[2 * img + 1];
  const double fy = (double)r * (h > 1 ? (double)(kPosGrid - 1) / (double)(h - 1) : 0.0);
  const double fx = (double)c * (w > 1 ? (double)(kPosGrid - 1) / (double)(w - 1) : 0.0);
  const int y0 = (int)floor(fy), x0 = (int)floor(fx);
  const int y1 = min(y0 + 1, kPosGrid - 1), x1 = min(x0 + 1, kPosGrid - 1);
  const double dy = fy - y0, dx = fx - x0;
  const double w00 = (1 - dy) * (1 - dx), w01 = (1 - dy) * dx, w10 = dy * (1 - dx), w11 = dy * dx;
  const int d0 = threadIdx.x * 8;
  float v00[8], v01[8], v10[8], v11[8];
  load8_bf16(table + (size_t)(y0 * kPosGrid + x0) * 1152 + d0, v00);
  load8_bf16(table + (size_t)(y0 * kPosGrid + x1) * 1152 + d0, v01);
  load8_bf16(table + (size_t)(y1 * kPosGrid + x0) * 1152 + d0, v10);
  load8_bf16(table + (size_t)(y1 * kPosGrid + x1) * 1152 + d0, v11);
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const double a = w00 * v00[2 * i] + w01 * v01[2 * i] + w10 * v10[2 * i] + w11 * v11[2 * i];
    const double b = w00 * v00[2 * i + 1] + w01 * v01[2 * i + 1] + w10 * v10[2 * i + 1] + w11 * v11[2 * i + 1];
    const __nv_bfloat16 ha = __double2bfloat16(a), hb = __double2bfloat16(b);
    o[i] = (uint32_t)__bfloat16_as_ushort(ha) | ((uint32_t)__bfloat16_as_ushort(hb) << 16);
  }
  *reinterpret_cast<uint4*>(out + (size_t)t * 1152 + d0) = make_uint4(o[0], o[1], o[2], o[3]);
}

// (row, col) of every patch of the packed images and the segment offsets
// ("Qwen3-VL-8B on RTX 5090", section 5: each image is its own attention window).
// Even grids are walked in 2x2-block order, so the merger's four neighbours are
// consecutive rows; odd grids row-major.
__global__ void positions_kernel(GridList grids, int n_total, int32_t* __restrict__ pos,
                                 int32_t* __restrict__ cu) {
  pdl_trigger();
  pdl_wait();
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t == 0) {
    int acc = 0;
    cu[0] = 0;
    for (int i = 0; i < grids.n; ++i) {
      acc += grids.hw[2 * i] * grids.hw[2 * i + 1];
      cu[i + 1] = acc;
    }
  }
  if (t >= n_total) return;
  int img, r, c;
  token_place(grids, t, img, r, c);
  pos[2 * t] = r;
  pos[2 * t + 1] = c;
}

// --------------------------------------------------------------- self-test
// Waits on an mbarrier that nothing ever arrives on, with a short limit: the
// wait gives up, raises the device error word and the kernel returns.  Used to
// check the timeout path without hanging anything.
__global__ void selftest_wait_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait_limit(smem_u32(&bar), 0, &abort_flag, limit_ns);
  __syncthreads();
}

}  // namespace

// ------------------------------------------------------------------ launchers

cudaError_t launch_selftest_wait(int limit_us, cudaStream_t st) {
  selftest_wait_kernel<<<1, 32, 0, st>>>((unsigned long long)limit_us * 1000ull);
  return cudaGetLastError();
}

template <int IT>
static void qa_launch(const __nv_bfloat16* x, int M, int K, int ldx, uint8_t* q, float* s, int lds,
                      cudaStream_t st) {
  const int threads = 128;
  launch_pdl(quant_act_kernel<IT>, dim3((unsigned)(((long long)M * 32 + threads - 1) / threads)), dim3(threads), 0,
             st, x, M, K, ldx, q, s, lds);
}

cudaError_t launch_quant_act(const __nv_bfloat16* x, int M, int K, int ldx, uint8_t* q, float* s,
                             int lds, cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  switch ((K + 255) / 256) {
#define VITQ_QA_CASE(N) \
  case N: qa_launch<N>(x, M, K, ldx, q, s, lds, st); break;
    VITQ_QA_CASE(1) VITQ_QA_CASE(2) VITQ_QA_CASE(3) VITQ_QA_CASE(4) VITQ_QA_CASE(5)
    VITQ_QA_CASE(6) VITQ_QA_CASE(7) VITQ_QA_CASE(8) VITQ_QA_CASE(9) VITQ_QA_CASE(10)
    VITQ_QA_CASE(11) VITQ_QA_CASE(12) VITQ_QA_CASE(13) VITQ_QA_CASE(14) VITQ_QA_CASE(15)
    VITQ_QA_CASE(16) VITQ_QA_CASE(17) VITQ_QA_CASE(18)
#undef VITQ_QA_CASE
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

template <int IT>
static void ln_launch(const __nv_bfloat16* x, int ldx, const __nv_bfloat16* g,
                      const __nv_bfloat16* b, int M, int K, double eps, uint8_t* q, float* s, int lds,
                      __nv_bfloat16* y, cudaStream_t st) {
  const dim3 grid((unsigned)((M + kLnRows - 1) / kLnRows)), block(16 * kLnRows);
  const size_t smem = (size_t)((K + 127) / 128) * 1536;
  auto kern = y ? ln_quant_kernel<IT, true> : ln_quant_kernel<IT, false>;
  if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  launch_pdl(kern, grid, block, smem, st, x, ldx, g, b, M, K, eps, q, s, lds, y);
}

cudaError_t launch_ln(const __nv_bfloat16* x, int ldx, const __nv_bfloat16* gamma, const __nv_bfloat16* beta,
                      int M, int K, double eps, uint8_t* q, float* s, int lds, __nv_bfloat16* y,
                      cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  const int chunks = (K + 127) / 128;
  switch (chunks) {
#define VITQ_LN_CASE(N) \
  case N: ln_launch<N>(x, ldx, gamma, beta, M, K, eps, q, s, lds, y, st); break;
    VITQ_LN_CASE(1) VITQ_LN_CASE(2) VITQ_LN_CASE(3) VITQ_LN_CASE(4) VITQ_LN_CASE(5)
    VITQ_LN_CASE(6) VITQ_LN_CASE(7) VITQ_LN_CASE(8) VITQ_LN_CASE(9)
#undef VITQ_LN_CASE
    default:
      if (chunks > kLnMaxChunks) return cudaErrorInvalidValue;
      ln_launch<0>(x, ldx, gamma, beta, M, K, eps, q, s, lds, y, st);
  }
  return cudaGetLastError();
}

cudaError_t build_gelu_table(cudaStream_t st) {
  gelu_table_kernel<<<256, 256, 0, st>>>();
  return cudaGetLastError();
}

cudaError_t launch_gelu(const __nv_bfloat16* f, int M, int K, int ldf, uint8_t* q, float* s, int lds,
                        __nv_bfloat16* y, int num_sms, cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(gelu_quant_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kGeluSmem);
  if (e != cudaSuccess) return e;
  const long long warps = (long long)M * ((K + 255) / 256);
  const long long ctas = (warps + kGeluThreads / 32 - 1) / (kGeluThreads / 32);
  return launch_pdl(gelu_quant_kernel, dim3((unsigned)(ctas < num_sms ? ctas : num_sms)), dim3(kGeluThreads),
                    kGeluSmem, st,
      f, M, K, ldf, q, s, lds, y);
}

cudaError_t launch_quant_weight(const __nv_bfloat16* w, int N, int K, uint8_t* q, float* s,
                                cudaStream_t st) {
  if (N == 0 || K == 0) return cudaSuccess;
  dim3 grid((K + 127) / 128, (N + 127) / 128);
  launch_pdl(quant_weight_kernel, grid, dim3(256), 0, st, w, N, K, q, s);
  return cudaGetLastError();
}

cudaError_t launch_rope_table(const int32_t* pos, int n, double theta, float* cs, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const int threads = 256;
  launch_pdl(rope_table_kernel, dim3((unsigned)(((long long)n * 36 + threads - 1) / threads)), dim3(threads), 0, st,
      pos, n, theta, cs);
  return cudaGetLastError();
}

cudaError_t launch_rope_apply(__nv_bfloat16* qkv, int n, const float* cs, int v_to_f16, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const long long items = (long long)n * kRopeItems;
  launch_pdl(rope_apply_kernel, dim3((unsigned)((items + 255) / 256)), dim3(256), 0, st, qkv, cs, n, v_to_f16);
  return cudaGetLastError();
}

cudaError_t launch_pos_interp(const GridList& g, int n_total, const __nv_bfloat16* table, __nv_bfloat16* out,
                              cudaStream_t st) {
  if (n_total == 0) return cudaSuccess;
  launch_pdl(pos_interp_kernel, dim3(n_total), dim3(144), 0, st, g, table, out);
  return cudaGetLastError();
}

cudaError_t launch_positions(const GridList& g, int n_total, int32_t* pos, int32_t* cu,
                             cudaStream_t st) {
  const int threads = 256;
  const int blocks = n_total > 0 ? (n_total + threads - 1) / threads : 1;
  launch_pdl(positions_kernel, dim3(blocks), dim3(threads), 0, st, g, n_total, pos, cu);
  return cudaGetLastError();
}

}  // namespace vitq

namespace vitq {
cudaError_t launch_ln_quant(const __nv_bfloat16* x, int ldx, const __nv_bfloat16* gamma,
                            const __nv_bfloat16* beta, int M, int K, double eps, uint8_t* q,
                            float* s, int lds, cudaStream_t st) {
  return launch_ln(x, ldx, gamma, beta, M, K, eps, q, s, lds, nullptr, st);
}
cudaError_t launch_gelu_quant(const __nv_bfloat16* f, int M, int K, int ldf, uint8_t* q, float* s,
                              int lds, int num_sms, cudaStream_t st) {
  return launch_gelu(f, M, K, ldf, q, s, lds, nullptr, num_sms, st);
}
}  // namespace vitq
