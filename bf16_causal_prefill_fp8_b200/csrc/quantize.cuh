// quantize.cuh -- the FP8 prepass: per-(batch, head) amax, scale = amax/448,
// e4m3 codes, with an optional 128-point Hadamard rotation of each row.
//
// Method: kongchang.com "Zyphra ZYFA", section "ZYFA 的性能与精度数据" (per-head
// scale factors map values into the e4m3 range) and spke.com "Zyphra ZYFA",
// accuracy section (quantizing Q, K and V is the main FP8 error source; a
// Hadamard rotation of Q and K roughly halves it).
//
// HBM-bound streaming passes.  A CTA covers whole sequence rows of one batch;
// every thread keeps kUnroll 16-byte loads in flight (the bytes in flight,
// not arithmetic, bound these kernels).
//
// Steps (all on `stream`; zyfa_quantize_qkv runs each step once for Q, K and
// V together, splitting the grid among them in proportion to their bytes):
//   1. memset(scale, 0)                         scale doubles as amax accumulator
//   2. quant_amax_kernel:  scale[b,h] = max(scale[b,h], max |x'|)   (fp32 bits,
//      atomicMax on the non-negative bit patterns, order-independent)
//   3. quant_codes_kernel: s = amax/448 (1 if amax == 0); code = e4m3(x'/s),
//      the quotient correctly rounded (div_by_scale)
//   4. quant_finalize_kernel: scale[b,h] = s
// x' is the row rotated by the orthonormal Sylvester transform when
// hadamard != 0 (stages of stride 1, 2, ..., 64 in fp32, then one multiply by
// fp32(2^-3.5)), else x itself.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

namespace zyfa {

// Programmatic dependent launch.  The prepass kernels after the first one
// are launched with programmatic stream serialization, so each may start
// while the kernel before it is still running.  griddep_wait blocks until
// that kernel has completed and its writes are visible (a no-op for a launch
// without the attribute); griddep_launch_dependents lets the next kernel
// start launching, whose CTAs then wait in griddep_wait before they touch
// this kernel's results.  The inputs x were written before the first prepass
// kernel, which launches in plain stream order, so reading them needs no wait.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

constexpr int kQuantThreads = 256;
constexpr int kUnroll = 4;        // rotated paths: rows in flight per warp
constexpr int kUnrollPlain = 4;   // plain paths: 16-byte loads in flight per thread
constexpr float kFwhtNorm = 0.08838834764831844055f;   // 2^-3.5 rounded to fp32

__device__ __forceinline__ uint16_t cvt_e4m3x2(float lo, float hi) {
  uint16_t d;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
  return d;
}

__device__ __forceinline__ float head_scale(float amax) {
  return amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
}

// x / s rounded to nearest even, given rc = RN(1/s) (Markstein's correction,
// P. Markstein, "Computation of elementary functions on the IBM RISC
// System/6000 processor", IBM J. Res. Dev. 34(1), 1990; also Muller et al.,
// "Handbook of Floating-Point Arithmetic", division by FMA): q0 = RN(x rc) is
// within one ulp of x/s, the residual x - s q0 is then exact in one FMA, and
// RN(q0 + residual * rc) is the correctly rounded quotient.  rc == 0 marks a
// scale too small or too large for the reciprocal to stay normal: plain
// division.  The quotients here are at most 448 in magnitude.
// FAST: every head of the CTA has a normal reciprocal, so the correction path
// runs alone (the CTA decides once; no division code in the loop).
template <bool FAST>
__device__ __forceinline__ float div_by_scale(float x, float s, float rc) {
  if (!FAST) return __fdiv_rn(x, s);
  const float q0 = __fmul_rn(x, rc);
  const float r = __fmaf_rn(-q0, s, x);
  return __fmaf_rn(r, rc, q0);
}

// Division by a runtime divisor d without a divide: m = ceil(2^64 / d)
// (m = 0 for d = 1), and for n < 2^32 the high word of n * m is floor(n / d)
// exactly (n m / 2^64 exceeds n / d by n (m - 2^64/d) / 2^64 < n / 2^64 < 1/d,
// which cannot carry the quotient past the next integer).  The kernels use it
// for the head index of a 16-byte vector, once per vector.
__host__ __device__ inline uint64_t div_magic(uint32_t d) { return d <= 1u ? 0ull : ~0ull / d + 1ull; }
__device__ __forceinline__ uint32_t div_by_magic(uint32_t n, uint64_t m) {
  return m ? static_cast<uint32_t>(__umul64hi(static_cast<uint64_t>(n), m)) : n;
}

__device__ __forceinline__ float scale_reciprocal(float s) {
  return (s >= 0x1p-120f && s <= 0x1p120f) ? __frcp_rn(s) : 0.0f;
}

// 16-byte vectors: 8 bf16 or 4 fp32 elements.
template <typename T> struct Vec;
template <> struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void unpack(const uint4& t, float* v) {
    v[0] = __uint_as_float(t.x << 16); v[1] = __uint_as_float(t.x & 0xffff0000u);
    v[2] = __uint_as_float(t.y << 16); v[3] = __uint_as_float(t.y & 0xffff0000u);
    v[4] = __uint_as_float(t.z << 16); v[5] = __uint_as_float(t.z & 0xffff0000u);
    v[6] = __uint_as_float(t.w << 16); v[7] = __uint_as_float(t.w & 0xffff0000u);
  }
};
template <> struct Vec<float> {
  static constexpr int N = 4;
  __device__ static void unpack(const uint4& t, float* v) {
    v[0] = __uint_as_float(t.x); v[1] = __uint_as_float(t.y);
    v[2] = __uint_as_float(t.z); v[3] = __uint_as_float(t.w);
  }
};

// Eight consecutive elements of a row as fp32 (one 16-byte bf16 load or two
// fp32 loads).  The rotation is defined by butterflies of stride 1, 2, 4, ...
// in that order, each stage the fp32 sum and difference of its pair; every
// layout below keeps that order.
template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&v)[8]);
template <>
__device__ __forceinline__ void load8<float>(const float* p, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[8]) {
  Vec<__nv_bfloat16>::unpack(__ldg(reinterpret_cast<const uint4*>(p)), v);
}

// Rotated rows of D = 128, four lanes per row: lane q of a quad holds
// elements 32q .. 32q+31 (four 16-byte bf16 / eight fp32 loads).  Butterflies
// of stride 1 .. 16 in registers, then 32 and 64 across the quad (lane xor 1,
// xor 2): two shuffles per element.
constexpr int kQuadRows = 1;   // rows in flight per quad lane
template <typename T>
__device__ __forceinline__ void load32(const T* p, float (&v)[32]) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    float t[8];
    load8<T>(p + 8 * c, t);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[8 * c + i] = t[i];
  }
}

__device__ __forceinline__ void fwht128_quad(float (&x)[32], int lq) {
  float a, b;
#pragma unroll
  for (int st = 1; st < 32; st <<= 1)
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if ((i & st) == 0) { a = x[i]; b = x[i + st]; x[i] = a + b; x[i + st] = a - b; }
#pragma unroll
  for (int sh = 1; sh < 4; sh <<= 1) {   // strides 32, 64
    const bool upper = (lq & sh) != 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float o = __shfl_xor_sync(0xffffffffu, x[i], sh);
      x[i] = upper ? (o - x[i]) : (x[i] + o);
    }
  }
#pragma unroll
  for (int i = 0; i < 32; ++i) x[i] = x[i] * kFwhtNorm;
}

// Rotated rows of D = 192 (MLA: H128 on dims 0..127, H64 on 128..191), one
// row per warp: lane l < 24 holds dims 8l .. 8l+7 (lanes 0-15 the 128-point
// block, 16-23 the 64-point block), lanes 24-31 zeros so every shuffle is
// full-mask.  Each block runs its own transform's stages in order (strides
// 1, 2, 4 in registers, then 8, 16, 32 across lanes, and 64 for the 128-point
// block only), then its own normalisation (2^-3.5, 2^-3).
__device__ __forceinline__ void fwht192_warp(float (&x)[8], int lane) {
  float a, b;
#pragma unroll
  for (int st = 1; st < 8; st <<= 1)
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if ((i & st) == 0) { a = x[i]; b = x[i + st]; x[i] = a + b; x[i + st] = a - b; }
  const bool b128 = lane < 16;
#pragma unroll
  for (int sh = 1; sh < 16; sh <<= 1) {   // strides 8, 16, 32 (both blocks), 64 (128-point block)
    const bool upper = (lane & sh) != 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float o = __shfl_xor_sync(0xffffffffu, x[i], sh);
      if (sh < 8 || b128) x[i] = upper ? (o - x[i]) : (x[i] + o);
    }
  }
  const float norm = b128 ? kFwhtNorm : 0.125f;
#pragma unroll
  for (int i = 0; i < 8; ++i) x[i] = x[i] * norm;
}

struct QuantArgs {
  const void* x;
  uint8_t* out;
  float* scale;            // [B*H]: amax accumulator, then the scales
  int S, H, D;
  int rows_per_cta;        // sequence rows of one batch per CTA
  uint64_t mg_vph;         // div_magic(16-byte vectors per head row: D / 8 bf16, D / 4 fp32)
  uint64_t mg_h;           // div_magic(H)
};

// The head of 16-byte vector vi of a chunk (chunks start on whole rows).
__device__ __forceinline__ uint32_t vec_head(const QuantArgs& a, uint32_t vi) {
  const uint32_t q = div_by_magic(vi, a.mg_vph);
  return q - static_cast<uint32_t>(a.H) * div_by_magic(q, a.mg_h);
}
// The head of row-vector v (one head's D elements) of a chunk.
__device__ __forceinline__ uint32_t row_head(const QuantArgs& a, uint32_t v) {
  return v - static_cast<uint32_t>(a.H) * div_by_magic(v, a.mg_h);
}

// Step 2 for sequence-row chunk `chunk` of batch b (one CTA); s_amax: [H].
template <typename T, bool HAD>
__device__ __forceinline__ void quant_amax_cta(const QuantArgs& a, int chunk, int b, unsigned int* s_amax) {
  griddep_launch_dependents();
  const int r0 = chunk * a.rows_per_cta, r1 = min(a.S, r0 + a.rows_per_cta);
  for (int h = threadIdx.x; h < a.H; h += blockDim.x) s_amax[h] = 0u;
  __syncthreads();
  const uint32_t HD = static_cast<uint32_t>(a.H) * a.D;
  const T* base = static_cast<const T*>(a.x) + (static_cast<size_t>(b) * a.S + r0) * HD;
  if (HAD && a.D == 192) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const int nrow = (r1 - r0) * a.H;
    for (int v0 = warp * kUnroll; v0 < nrow; v0 += nw * kUnroll) {
      float x[kUnroll][8];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        if (v0 + u < nrow && lane < 24) load8<T>(base + static_cast<size_t>(v0 + u) * 192 + 8 * lane, x[u]);
        else
#pragma unroll
          for (int i = 0; i < 8; ++i) x[u][i] = 0.0f;
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        if (v0 + u >= nrow) break;
        fwht192_warp(x[u], lane);
        float mx = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) mx = fmaxf(mx, fabsf(x[u][i]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (lane == 0) atomicMax(&s_amax[row_head(a, v0 + u)], __float_as_uint(mx));
      }
    }
  } else if (HAD) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const int quad = lane >> 2, lq = lane & 3;
    const int nvec = (r1 - r0) * a.H;          // 128-element rows, 8 per warp and step
    for (int v0 = warp * 8 * kQuadRows; v0 < nvec; v0 += nw * 8 * kQuadRows) {
      float x[kQuadRows][32];
#pragma unroll
      for (int u = 0; u < kQuadRows; ++u) {
        const int v = v0 + 8 * u + quad;
        if (v < nvec) load32<T>(base + static_cast<size_t>(v) * 128 + 32 * lq, x[u]);
        else
#pragma unroll
          for (int i = 0; i < 32; ++i) x[u][i] = 0.0f;
      }
#pragma unroll
      for (int u = 0; u < kQuadRows; ++u) {
        if (v0 + 8 * u >= nvec) break;                  // every row of the step past the end
        fwht128_quad(x[u], lq);
        float mx = 0.0f;
#pragma unroll
        for (int i = 0; i < 32; ++i) mx = fmaxf(mx, fabsf(x[u][i]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const int v = v0 + 8 * u + quad;
        if (lq == 0 && v < nvec) atomicMax(&s_amax[row_head(a, v)], __float_as_uint(mx));
      }
    }
  } else {
    constexpr int N = Vec<T>::N;
    const uint32_t vpr = HD / N;                       // 16-byte vectors per row
    const uint32_t nvec = static_cast<uint32_t>(r1 - r0) * vpr;
    const uint4* src = reinterpret_cast<const uint4*>(base);
    for (uint32_t v0 = threadIdx.x; v0 < nvec; v0 += blockDim.x * kUnrollPlain) {
      uint4 raw[kUnrollPlain];
#pragma unroll
      for (int u = 0; u < kUnrollPlain; ++u) {
        const uint32_t vi = v0 + u * blockDim.x;
        if (vi < nvec) raw[u] = __ldg(src + vi);
      }
#pragma unroll
      for (int u = 0; u < kUnrollPlain; ++u) {
        const uint32_t vi = v0 + u * blockDim.x;
        if (vi >= nvec) break;
        float x[N];
        Vec<T>::unpack(raw[u], x);
        float mx = 0.0f;
#pragma unroll
        for (int i = 0; i < N; ++i) mx = fmaxf(mx, fabsf(x[i]));
        atomicMax(&s_amax[vec_head(a, vi)], __float_as_uint(mx));
      }
    }
  }
  __syncthreads();
  griddep_wait();   // the scale array holds zeros (the zero step has completed)
  for (int h = threadIdx.x; h < a.H; h += blockDim.x)
    atomicMax(reinterpret_cast<unsigned int*>(a.scale) + static_cast<size_t>(b) * a.H + h, s_amax[h]);
}

// Step 3 for one chunk; reads the finished amax of each (b, h); s_sc: [H].
template <typename T, bool HAD, bool FAST>
__device__ __forceinline__ void quant_codes_loop(const QuantArgs& a, int r0, int r1, int b, const float* s_sc,
                                                 const float* s_rc) {
  const uint32_t HD = static_cast<uint32_t>(a.H) * a.D;
  const size_t off = (static_cast<size_t>(b) * a.S + r0) * HD;
  const T* base = static_cast<const T*>(a.x) + off;
  uint8_t* obase = a.out + off;
  if (HAD && a.D == 192) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const int nrow = (r1 - r0) * a.H;
    for (int v0 = warp * kUnroll; v0 < nrow; v0 += nw * kUnroll) {
      float x[kUnroll][8];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        if (v0 + u < nrow && lane < 24) load8<T>(base + static_cast<size_t>(v0 + u) * 192 + 8 * lane, x[u]);
        else
#pragma unroll
          for (int i = 0; i < 8; ++i) x[u][i] = 0.0f;
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        if (v0 + u >= nrow) break;
        fwht192_warp(x[u], lane);
        if (lane >= 24) continue;
        const int hh = row_head(a, v0 + u);
        const float sc = s_sc[hh], rc = s_rc[hh];
        uint32_t w[2];
#pragma unroll
        for (int i = 0; i < 2; ++i)
          w[i] = cvt_e4m3x2(div_by_scale<FAST>(x[u][4 * i], sc, rc), div_by_scale<FAST>(x[u][4 * i + 1], sc, rc)) |
                 (static_cast<uint32_t>(cvt_e4m3x2(div_by_scale<FAST>(x[u][4 * i + 2], sc, rc),
                                                   div_by_scale<FAST>(x[u][4 * i + 3], sc, rc))) << 16);
        *reinterpret_cast<uint2*>(obase + static_cast<size_t>(v0 + u) * 192 + 8 * lane) = make_uint2(w[0], w[1]);
      }
    }
  } else if (HAD) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const int quad = lane >> 2, lq = lane & 3;
    const int nvec = (r1 - r0) * a.H;
    for (int v0 = warp * 8 * kQuadRows; v0 < nvec; v0 += nw * 8 * kQuadRows) {
      float x[kQuadRows][32];
#pragma unroll
      for (int u = 0; u < kQuadRows; ++u) {
        const int v = v0 + 8 * u + quad;
        if (v < nvec) load32<T>(base + static_cast<size_t>(v) * 128 + 32 * lq, x[u]);
        else
#pragma unroll
          for (int i = 0; i < 32; ++i) x[u][i] = 0.0f;
      }
#pragma unroll
      for (int u = 0; u < kQuadRows; ++u) {
        if (v0 + 8 * u >= nvec) break;
        fwht128_quad(x[u], lq);
        const int v = v0 + 8 * u + quad;
        if (v >= nvec) continue;
        const int hh = row_head(a, v);
        const float sc = s_sc[hh], rc = s_rc[hh];
        uint32_t w[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
          w[i] = cvt_e4m3x2(div_by_scale<FAST>(x[u][4 * i], sc, rc), div_by_scale<FAST>(x[u][4 * i + 1], sc, rc)) |
                 (static_cast<uint32_t>(cvt_e4m3x2(div_by_scale<FAST>(x[u][4 * i + 2], sc, rc),
                                                   div_by_scale<FAST>(x[u][4 * i + 3], sc, rc))) << 16);
        uint4* dst = reinterpret_cast<uint4*>(obase + static_cast<size_t>(v) * 128 + 32 * lq);
        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
      }
    }
  } else {
    constexpr int N = Vec<T>::N;
    const uint32_t vpr = HD / N;
    const uint32_t nvec = static_cast<uint32_t>(r1 - r0) * vpr;
    const uint4* src = reinterpret_cast<const uint4*>(base);
    for (uint32_t v0 = threadIdx.x; v0 < nvec; v0 += blockDim.x * kUnrollPlain) {
      uint4 raw[kUnrollPlain];
#pragma unroll
      for (int u = 0; u < kUnrollPlain; ++u) {
        const uint32_t vi = v0 + u * blockDim.x;
        if (vi < nvec) raw[u] = __ldg(src + vi);
      }
#pragma unroll
      for (int u = 0; u < kUnrollPlain; ++u) {
        const uint32_t vi = v0 + u * blockDim.x;
        if (vi >= nvec) break;
        float x[N];
        Vec<T>::unpack(raw[u], x);
        const uint32_t hh = vec_head(a, vi);
        const float sc = s_sc[hh], rc = s_rc[hh];
        uint32_t w[N / 4];
#pragma unroll
        for (int i = 0; i < N / 4; ++i)
          w[i] = cvt_e4m3x2(div_by_scale<FAST>(x[4 * i], sc, rc), div_by_scale<FAST>(x[4 * i + 1], sc, rc)) |
                 (static_cast<uint32_t>(cvt_e4m3x2(div_by_scale<FAST>(x[4 * i + 2], sc, rc),
                                                   div_by_scale<FAST>(x[4 * i + 3], sc, rc))) << 16);
        if constexpr (N == 8) *reinterpret_cast<uint2*>(obase + static_cast<size_t>(vi) * 8) = make_uint2(w[0], w[1]);
        else *reinterpret_cast<uint32_t*>(obase + static_cast<size_t>(vi) * 4) = w[0];
      }
    }
  }
}

template <typename T, bool HAD>
__device__ __forceinline__ void quant_codes_cta(const QuantArgs& a, int chunk, int b, float* s_sc) {
  griddep_launch_dependents();
  griddep_wait();   // every amax of the step is final
  const int r0 = chunk * a.rows_per_cta, r1 = min(a.S, r0 + a.rows_per_cta);
  float* s_rc = s_sc + a.H;   // RN(1 / scale) per head
  int fast = 1;
  for (int h = threadIdx.x; h < a.H; h += blockDim.x) {
    const float sc = head_scale(a.scale[static_cast<size_t>(b) * a.H + h]);
    const float rc = scale_reciprocal(sc);
    s_sc[h] = sc;
    s_rc[h] = rc;
    if (rc == 0.0f) fast = 0;
  }
  if (__syncthreads_and(fast)) quant_codes_loop<T, HAD, true>(a, r0, r1, b, s_sc, s_rc);
  else quant_codes_loop<T, HAD, false>(a, r0, r1, b, s_sc, s_rc);
}

// One tensor: grid = (ceil(S / rows_per_cta), B), block = kQuantThreads,
// dynamic shared memory H * 8 bytes.
template <typename T, bool HAD>
__global__ void __launch_bounds__(kQuantThreads) quant_amax_kernel(QuantArgs a) {
  extern __shared__ unsigned int s_amax[];
  quant_amax_cta<T, HAD>(a, blockIdx.x, blockIdx.y, s_amax);
}
template <typename T, bool HAD>
__global__ void __launch_bounds__(kQuantThreads) quant_codes_kernel(QuantArgs a) {
  extern __shared__ float s_sc[];
  quant_codes_cta<T, HAD>(a, blockIdx.x, blockIdx.y, s_sc);
}

// Step 4.
__global__ void quant_finalize_kernel(float* scale, int n) {
  griddep_wait();   // every codes CTA has read the amax
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) scale[i] = head_scale(scale[i]);
}

// Q, K and V in one launch per step: the CTAs of grid column x belong to
// tensor i for first[i] <= x < first[i + 1] (chunk x - first[i]); had[i]
// selects the rotated path.  Shared memory: max H * 8 bytes.
struct Quant3Args {
  QuantArgs t[3];
  int had[3];
  int first[4];
};

__device__ __forceinline__ int quant3_pick(const Quant3Args& a, int x) {
  return x < a.first[1] ? 0 : (x < a.first[2] ? 1 : 2);
}

template <typename T>
__global__ void __launch_bounds__(kQuantThreads) quant3_amax_kernel(const __grid_constant__ Quant3Args a) {
  extern __shared__ unsigned int s_amax[];
  const int i = quant3_pick(a, blockIdx.x), chunk = blockIdx.x - a.first[i];
  if (a.had[i]) quant_amax_cta<T, true>(a.t[i], chunk, blockIdx.y, s_amax);
  else quant_amax_cta<T, false>(a.t[i], chunk, blockIdx.y, s_amax);
}

template <typename T>
__global__ void __launch_bounds__(kQuantThreads) quant3_codes_kernel(const __grid_constant__ Quant3Args a) {
  extern __shared__ float s_sc[];
  const int i = quant3_pick(a, blockIdx.x), chunk = blockIdx.x - a.first[i];
  if (a.had[i]) quant_codes_cta<T, true>(a.t[i], chunk, blockIdx.y, s_sc);
  else quant_codes_cta<T, false>(a.t[i], chunk, blockIdx.y, s_sc);
}

// Variable-length batch: tensors packed [T, H, D], sequence s at rows
// cu[s] .. cu[s+1]-1 with its own scale per head ([nseq, H] per tensor).
// Tensor i's CTAs (grid columns first[i] .. first[i+1]-1) enumerate the
// chunks of every sequence in order, ceil(len / rows_per_cta) per sequence,
// so no CTA is idle; each runs the fixed-length step on its sequence alone
// (base and scale pointers moved to it, S = its length).
constexpr int kMaxQuantSeqs = 384;
struct Quant3VarArgs {
  Quant3Args q;                  // t[i].S unused; rows_per_cta per tensor
  int n;                         // sequences
  int cu[kMaxQuantSeqs + 1];
};
static_assert(sizeof(Quant3VarArgs) <= 4096, "kernel parameter space");

template <typename T>
__device__ __forceinline__ bool quant3v_select(const Quant3VarArgs& a, QuantArgs& t, int& i, int& chunk) {
  i = quant3_pick(a.q, blockIdx.x);
  t = a.q.t[i];
  // the sequence this chunk belongs to: a scan over the sequences' chunk
  // counts (every thread takes the same path)
  int c = blockIdx.x - a.q.first[i], s = 0;
  for (; s < a.n; ++s) {
    const int nch = (a.cu[s + 1] - a.cu[s] + t.rows_per_cta - 1) / t.rows_per_cta;
    if (c < nch) break;
    c -= nch;
  }
  if (s >= a.n) return false;   // past the last chunk (the host sizes the grid exactly)
  chunk = c;
  const int r0 = a.cu[s], len = a.cu[s + 1] - r0;
  const size_t off = static_cast<size_t>(r0) * t.H * t.D;
  t.x = static_cast<const T*>(t.x) + off;
  t.out += off;
  t.scale += static_cast<size_t>(s) * t.H;
  t.S = len;
  return true;
}

template <typename T>
__global__ void __launch_bounds__(kQuantThreads) quant3v_amax_kernel(const __grid_constant__ Quant3VarArgs a) {
  extern __shared__ unsigned int s_amax[];
  QuantArgs t;
  int i, chunk;
  if (!quant3v_select<T>(a, t, i, chunk)) return;
  if (a.q.had[i]) quant_amax_cta<T, true>(t, chunk, 0, s_amax);
  else quant_amax_cta<T, false>(t, chunk, 0, s_amax);
}

template <typename T>
__global__ void __launch_bounds__(kQuantThreads) quant3v_codes_kernel(const __grid_constant__ Quant3VarArgs a) {
  extern __shared__ float s_sc[];
  QuantArgs t;
  int i, chunk;
  if (!quant3v_select<T>(a, t, i, chunk)) return;
  if (a.q.had[i]) quant_codes_cta<T, true>(t, chunk, 0, s_sc);
  else quant_codes_cta<T, false>(t, chunk, 0, s_sc);
}

// Steps 1 and 4 for the three scale arrays (n[i] = B * H_i entries each).
__global__ void quant3_zero_kernel(float* s0, float* s1, float* s2, int n0, int n1, int n2) {
  griddep_launch_dependents();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n0) s0[i] = 0.0f;
  else if (i < n0 + n1) s1[i - n0] = 0.0f;
  else if (i < n0 + n1 + n2) s2[i - n0 - n1] = 0.0f;
}
__global__ void quant3_finalize_kernel(float* s0, float* s1, float* s2, int n0, int n1, int n2) {
  griddep_wait();   // every codes CTA has read the amax
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  float* p = i < n0 ? s0 + i : (i < n0 + n1 ? s1 + (i - n0) : s2 + (i - n0 - n1));
  if (i < n0 + n1 + n2) *p = head_scale(*p);
}

}  // namespace zyfa
