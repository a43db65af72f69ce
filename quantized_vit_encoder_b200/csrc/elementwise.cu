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

// The quotient y / s that decides an E4M3 code.  The code depends only on which
// side of an E4M3 rounding midpoint fl(y / s) lies; y * fl(1 / s) is within a
// few ulps of fl(y / s), so the exact IEEE division is taken only when that
// product lies within 16 ulps of a midpoint (mantissa tail 0x80000) or below
// the normal E4M3 range.  The result therefore always encodes like fl(y / s).
__device__ __forceinline__ float e4m3_quotient(float y, float s, float r) {
  float q = y * r;
  const uint32_t b = __float_as_uint(q) & 0x7FFFFFFFu;
  // mantissa tail within 16 of 0x80000  <=>  ((b - 0x7FFF0) mod 2^20) <= 32
  if (b < 0x3C800000u || ((b - 0x7FFF0u) & 0xFFFFFu) <= 32u) q = __fdiv_rn(y, s);
  return q;
}

// Quantise 8 consecutive values of one 128-column group given the group scale.
// A scale below the fp32 normal range (amax < 448 * 2^-126) has no finite
// reciprocal; those groups always divide exactly.
__device__ __forceinline__ uint2 quant8(const float (&v)[8], float s) {
  uint32_t c[4] = {0u, 0u, 0u, 0u};
  if (s >= 1.17549435e-38f) {
    const float r = __frcp_rn(s);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      c[i] = cvt_e4m3x2(e4m3_quotient(v[2 * i], s, r), e4m3_quotient(v[2 * i + 1], s, r));
  } else if (s > 0.f) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      c[i] = cvt_e4m3x2(__fdiv_rn(v[2 * i], s), __fdiv_rn(v[2 * i + 1], s));
  }
  return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

// Max over the 16 lanes of a half warp.
__device__ __forceinline__ float half_warp_max(float v) {
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
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

// Exact value of a bf16 bit pattern as fp64, by moving its fields (zero and
// bf16 subnormals, below 1.2e-38, give 0).
__device__ __forceinline__ double bf16_bits_to_f64(uint32_t h) {
  const uint32_t e = (h >> 7) & 0xFFu;
  uint64_t bits = (uint64_t)(h & 0x8000u) << 48;
  if (e) bits |= ((uint64_t)(e + 896u) << 52) | ((uint64_t)(h & 0x7Fu) << 45);
  return __longlong_as_double((long long)bits);
}

// Lane layout shared by the row kernels: a warp covers 256 columns per step;
// lanes 0-15 hold group 2*step, lanes 16-31 group 2*step+1, 8 columns each.
__device__ __forceinline__ int lane_col(int step, int lane) { return step * 256 + lane * 8; }

// Group amax over the half warp, scale, codes and scale store for one step.
__device__ __forceinline__ void quant_store(const float (&v)[8], bool ok, int lane, int row, int col, int K,
                                            uint8_t* __restrict__ q, float* __restrict__ s, int lds) {
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(v[i]));
  a = half_warp_max(a);
  const float sc = __fdiv_rn(a, kE4M3Max);
  if (ok) {
    *reinterpret_cast<uint2*>(q + (size_t)row * K + col) = quant8(v, sc);
    if ((lane & 15) == 0) s[(size_t)(col >> 7) * lds + row] = sc;
  }
}

// ------------------------------------------------------------ activation quant
// One warp per row; every load of the row is issued before any use.

template <int ITERS>
__global__ void quant_act_kernel(const __nv_bfloat16* __restrict__ x, int M, int K, int ldx,
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
    float v[8];
    unpack8(raw[it], v);
    quant_store(v, col < K, lane, row, col, K, q, s, lds);
  }
}

// --------------------------------------------------------- LayerNorm + quant
// One warp per row, eight rows per CTA; gamma and beta are staged once per CTA
// in shared memory.  The statistics are exact fp64 sums of the bf16 inputs
// (sum and sum of squares); the normalised value is evaluated in fp32 and,
// when it lies within its error bound of a bf16 rounding midpoint, recomputed
// in fp64, so the bf16 result is the rounding of the fp64 value
// (x - mean) * rstd * gamma + beta.

constexpr int kLnRows = 8;

template <int ITERS, bool kOutBf16>
__global__ void __launch_bounds__(32 * kLnRows, 3)
    ln_quant_kernel(const __nv_bfloat16* __restrict__ x, int ldx, const __nv_bfloat16* __restrict__ gamma,
                    const __nv_bfloat16* __restrict__ beta, int M, int K, double eps,
                    uint8_t* __restrict__ q, float* __restrict__ s, int lds, __nv_bfloat16* __restrict__ y) {
  __shared__ uint4 sg[ITERS * 32], sb[ITERS * 32];
  pdl_trigger();
  for (int i = threadIdx.x; i < ITERS * 32; i += blockDim.x) {
    const int col = lane_col(i >> 5, i & 31);
    sg[i] = col < K ? *reinterpret_cast<const uint4*>(gamma + col) : make_uint4(0, 0, 0, 0);
    sb[i] = col < K ? *reinterpret_cast<const uint4*>(beta + col) : make_uint4(0, 0, 0, 0);
  }
  __syncthreads();
  pdl_wait();   // x may be the previous kernel's output
  const int row = blockIdx.x * kLnRows + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  // Rows of up to 8 steps stay in registers; wider rows (the merger's 4608) are
  // read again from L1/L2 in the second pass.
  constexpr bool kKeep = ITERS <= 8;
  constexpr int kHeld = kKeep ? ITERS : 1;
  const __nv_bfloat16* xr = x + (size_t)row * ldx;
  auto load_step = [&](int it) {
    const int col = lane_col(it, lane);
    return col < K ? *reinterpret_cast<const uint4*>(xr + col) : make_uint4(0, 0, 0, 0);
  };
  uint4 raw[kHeld];
  if (kKeep) {
#pragma unroll
    for (int it = 0; it < kHeld; ++it) raw[it] = load_step(it);
  }
  // exact fp64 sums of the bf16 inputs (bf16 -> fp32 -> fp64 is exact); 2 chains each
  double s1[2] = {0.0, 0.0}, s2[2] = {0.0, 0.0};
#pragma unroll
  for (int it = 0; it < ITERS; ++it) {
    float v[8];
    unpack8(kKeep ? raw[kKeep ? it : 0] : load_step(it), v);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const double d = (double)v[i];
      s1[i & 1] += d;
      s2[i & 1] = fma(d, d, s2[i & 1]);
    }
  }
  double t1 = s1[0] + s1[1], t2 = s2[0] + s2[1];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    t1 += __shfl_xor_sync(0xffffffffu, t1, o);
    t2 += __shfl_xor_sync(0xffffffffu, t2, o);
  }
  const double mean = t1 / (double)K;
  const double var = fmax(t2 / (double)K - mean * mean, 0.0);
  const double rstd = 1.0 / sqrt(var + eps);
  const float mh = (float)mean, ml = (float)(mean - (double)mh), r32 = (float)rstd;
#pragma unroll
  for (int it = 0; it < ITERS; ++it) {
    const int col = lane_col(it, lane);
    const bool ok = col < K;
    const uint4 rv = kKeep ? raw[kKeep ? it : 0] : load_step(it);
    float v[8];
    unpack8(rv, v);
    if (ok) {
      float g[8], b[8];
      unpack8(sg[it * 32 + lane], g);
      unpack8(sb[it * 32 + lane], b);
      bool slow = false;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float t = ((v[i] - mh) - ml) * r32;
        const float y = fmaf(t, g[i], b[i]);
        // fp32 error of y is below (|t g| + |b|) 2^-20; distance of y to the nearest
        // bf16 rounding midpoint = half a bf16 ulp (from y's exponent) - |y - bf16(y)|
        const float yr = __bfloat162float(__float2bfloat16_rn(y));
        const float half = __uint_as_float((__float_as_uint(y) & 0x7F800000u) - (8u << 23));
        const float err = (fabsf(t * g[i]) + fabsf(b[i])) * 9.5367431640625e-07f;
        slow |= (half - fabsf(y - yr) <= err) | (fabsf(y) < 1e-30f);
        v[i] = yr;
      }
      if (slow) {   // rare: redo the flagged values in fp64 from the inputs
        float xi[8];
        unpack8(rv, xi);
        unpack8(sg[it * 32 + lane], g);
        unpack8(sb[it * 32 + lane], b);
#pragma unroll 1
        for (int i = 0; i < 8; ++i) {
          const float t = ((xi[i] - mh) - ml) * r32;
          const float y = fmaf(t, g[i], b[i]);
          const float yr = __bfloat162float(__float2bfloat16_rn(y));
          const float half = __uint_as_float((__float_as_uint(y) & 0x7F800000u) - (8u << 23));
          const float err = (fabsf(t * g[i]) + fabsf(b[i])) * 9.5367431640625e-07f;
          if (half - fabsf(y - yr) <= err || fabsf(y) < 1e-30f) {
            const double yd = ((double)xi[i] - mean) * rstd * (double)g[i] + (double)b[i];
            v[i] = __bfloat162float(__double2bfloat16(yd));
          }
        }
      }
    }
    if (kOutBf16) {   // bf16 output (the bf16 blocks and mergers): values are already bf16
      if (ok)
        *reinterpret_cast<uint4*>(y + (size_t)row * K + col) =
            make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                       pack_bf16x2(v[6], v[7]));
    } else {
      quant_store(v, ok, lane, row, col, K, q, s, lds);
    }
  }
}

// ------------------------------------------------------------- GELU + quant
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
// takes (row, 256-column step) items in turn (lane layout of lane_col).
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
  const int items = M * steps;
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * (kGeluThreads / 32);
  // each warp walks items w, w + warps, ...; the next item's 8 inputs per lane are
  // loaded before the current item is processed, so the load latency overlaps the work
  auto load = [&](int w) {
    const int row = w / steps, col = lane_col(w - row * steps, lane);
    return (w < items && col < K) ? *reinterpret_cast<const uint4*>(f + (size_t)row * ldf + col)
                                  : make_uint4(0u, 0u, 0u, 0u);
  };
  int w = blockIdx.x * (kGeluThreads / 32) + (threadIdx.x >> 5);
  uint4 cur = load(w);
  for (; w < items; w += warps) {
    const uint4 nxt = load(w + warps);
    const int row = w / steps;
    const int st = w - row * steps;
    const int col = lane_col(st, lane);
    const bool ok = col < K;
    float v[8];
    const uint32_t wd[4] = {cur.x, cur.y, cur.z, cur.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {   // zero inputs (past K) read GELU(0) = 0
      v[2 * i] = __uint_as_float((uint32_t)lut[wd[i] & 0xFFFFu] << 16);
      v[2 * i + 1] = __uint_as_float((uint32_t)lut[wd[i] >> 16] << 16);
    }
    if (y) {   // bf16 output (may be f itself: each lane reads its 8 values before writing them)
      if (ok)
        *reinterpret_cast<uint4*>(y + (size_t)row * ldf + col) =
            make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                       pack_bf16x2(v[6], v[7]));
    } else {
      quant_store(v, ok, lane, row, col, K, q, s, lds);
    }
    cur = nxt;
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

// One CTA per token, one thread per 8-element chunk.  Chunks 0..287 are the
// token's q and k heads (9 per head): x'_j = x_j c_j - x_(j+36) s_j,
// x'_(j+36) = x_(j+36) c_j + x_j s_j; the partner elements of chunk cc live in
// two neighbouring chunks A (elements 4..7) and B (elements 0..3).  Chunks
// 288..431 are the v heads, converted to fp16 in place when v_to_f16 (round to
// nearest: exact for 2^-14 <= |v| < 65504, within 2^-25 below).  All reads happen before the barrier and all
// writes after it, so the in-place update never reads a rotated value.
__global__ void __launch_bounds__(432) rope_apply_kernel(__nv_bfloat16* __restrict__ qkv,
                                                         const float* __restrict__ cs, int v_to_f16) {
  pdl_trigger();
  pdl_wait();
  const int t = blockIdx.x;
  const int c = threadIdx.x;
  __nv_bfloat16* base = qkv + (size_t)t * 3456;
  uint4 out = make_uint4(0, 0, 0, 0);
  __nv_bfloat16* dst = nullptr;
  if (c < 288) {
    const int slot = c / 9, cc = c - slot * 9;
    const __nv_bfloat16* head = base + slot * 72;
    int ca, cb, k0, k1;   // partner chunks, cos/sin offsets of elements 0..3 and 4..7
    if (cc < 4) {
      ca = cc + 4; cb = cc + 5; k0 = 8 * cc; k1 = 8 * cc + 4;
    } else if (cc == 4) {
      ca = 8; cb = 0; k0 = 32; k1 = 0;
    } else {
      ca = cc - 5; cb = cc - 4; k0 = 8 * cc - 36; k1 = 8 * cc - 32;
    }
    float x[8], pa[8], pb[8];
    load8_bf16(head + cc * 8, x);
    load8_bf16(head + ca * 8, pa);
    load8_bf16(head + cb * 8, pb);
    const float* tc = cs + (size_t)t * 72;
    const float4 c0 = __ldg(reinterpret_cast<const float4*>(tc + k0));
    const float4 c1 = __ldg(reinterpret_cast<const float4*>(tc + k1));
    const float4 s0 = __ldg(reinterpret_cast<const float4*>(tc + 36 + k0));
    const float4 s1 = __ldg(reinterpret_cast<const float4*>(tc + 36 + k1));
    const float cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
    const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
    const float pv[8] = {pa[4], pa[5], pa[6], pa[7], pb[0], pb[1], pb[2], pb[3]};
    float o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const bool first_half = cc < 4 || (cc == 4 && i < 4);   // element j < 36
      o[i] = first_half ? fmaf(x[i], cv[i], -pv[i] * sv[i]) : fmaf(x[i], cv[i], pv[i] * sv[i]);
    }
    out.x = pack_bf16x2(o[0], o[1]);
    out.y = pack_bf16x2(o[2], o[3]);
    out.z = pack_bf16x2(o[4], o[5]);
    out.w = pack_bf16x2(o[6], o[7]);
    dst = base + slot * 72 + cc * 8;
  } else if (v_to_f16) {
    dst = base + 2304 + (c - 288) * 8;
    float v[8];
    load8_bf16(dst, v);
    __half2 h0 = __floats2half2_rn(v[0], v[1]), h1 = __floats2half2_rn(v[2], v[3]);
    __half2 h2 = __floats2half2_rn(v[4], v[5]), h3 = __floats2half2_rn(v[6], v[7]);
    out.x = *reinterpret_cast<uint32_t*>(&h0);
    out.y = *reinterpret_cast<uint32_t*>(&h1);
    out.z = *reinterpret_cast<uint32_t*>(&h2);
    out.w = *reinterpret_cast<uint32_t*>(&h3);
  }
  __syncthreads();
  if (dst) *reinterpret_cast<uint4*>(dst) = out;
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
  if (y)
    launch_pdl(ln_quant_kernel<IT, true>, dim3((unsigned)((M + kLnRows - 1) / kLnRows)), dim3(32 * kLnRows), 0, st,
               x, ldx, g, b, M, K, eps, q, s, lds, y);
  else
    launch_pdl(ln_quant_kernel<IT, false>, dim3((unsigned)((M + kLnRows - 1) / kLnRows)), dim3(32 * kLnRows), 0, st,
               x, ldx, g, b, M, K, eps, q, s, lds, y);
}

cudaError_t launch_ln(const __nv_bfloat16* x, int ldx, const __nv_bfloat16* gamma, const __nv_bfloat16* beta,
                      int M, int K, double eps, uint8_t* q, float* s, int lds, __nv_bfloat16* y,
                      cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  const int it = (K + 255) / 256;
  switch (it) {
#define VITQ_LN_CASE(N) \
  case N: ln_launch<N>(x, ldx, gamma, beta, M, K, eps, q, s, lds, y, st); break;
    VITQ_LN_CASE(1) VITQ_LN_CASE(2) VITQ_LN_CASE(3) VITQ_LN_CASE(4) VITQ_LN_CASE(5)
    VITQ_LN_CASE(6) VITQ_LN_CASE(7) VITQ_LN_CASE(8) VITQ_LN_CASE(9) VITQ_LN_CASE(10)
    VITQ_LN_CASE(11) VITQ_LN_CASE(12) VITQ_LN_CASE(13) VITQ_LN_CASE(14) VITQ_LN_CASE(15)
    VITQ_LN_CASE(16) VITQ_LN_CASE(17) VITQ_LN_CASE(18)
#undef VITQ_LN_CASE
    default: return cudaErrorInvalidValue;
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
  launch_pdl(rope_apply_kernel, dim3(n), dim3(432), 0, st, qkv, cs, v_to_f16);
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
