// Shared device helpers of the dispatch/combine kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_dc.h"

namespace moe {

constexpr int kMaxK = 16;
constexpr int kVecElems = 8;  // 16-bit values per 16-byte vector

// ---- 16-bit float traits: exact widening, round-to-nearest-even narrowing ----

struct Bf16 {
  static __device__ __forceinline__ float2 widen2(uint32_t u) {
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
  }
  static __device__ __forceinline__ uint32_t narrow2(float lo, float hi) {
    __nv_bfloat162 r = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&r);
  }
};

// Running max of |value| over 16-bit pairs, kept packed (one instruction per
// pair of values); max and abs are exact, so the widened result equals the
// fp32 max of the widened values.
struct Bf16Abs {
  static __device__ __forceinline__ uint32_t absmax2(uint32_t acc, uint32_t v) {
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&acc);
    __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&v);
    __nv_bfloat162 r = __hmax2(a, __habs2(b));
    return *reinterpret_cast<uint32_t*>(&r);
  }
};

struct Fp16 {
  static __device__ __forceinline__ float2 widen2(uint32_t u) {
    __half2 h = *reinterpret_cast<__half2*>(&u);
    return __half22float2(h);
  }
  static __device__ __forceinline__ uint32_t narrow2(float lo, float hi) {
    __half2 r = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&r);
  }
};

template <typename T>
__device__ __forceinline__ void widen8(const uint4& v, float (&f)[8]) {
  float2 a = T::widen2(v.x), b = T::widen2(v.y), c = T::widen2(v.z), d = T::widen2(v.w);
  f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
  f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}

template <typename T>
__device__ __forceinline__ uint4 narrow8(const float (&f)[8]) {
  uint4 v;
  v.x = T::narrow2(f[0], f[1]);
  v.y = T::narrow2(f[2], f[3]);
  v.z = T::narrow2(f[4], f[5]);
  v.w = T::narrow2(f[6], f[7]);
  return v;
}

// Packed running max of |x| over a 16-byte vector (8 values), per dtype.
template <typename T>
__device__ __forceinline__ uint32_t absmax_v4(uint32_t acc, const uint4& v);
template <>
__device__ __forceinline__ uint32_t absmax_v4<Bf16>(uint32_t acc, const uint4& v) {
  acc = Bf16Abs::absmax2(acc, v.x);
  acc = Bf16Abs::absmax2(acc, v.y);
  acc = Bf16Abs::absmax2(acc, v.z);
  return Bf16Abs::absmax2(acc, v.w);
}
template <>
__device__ __forceinline__ uint32_t absmax_v4<Fp16>(uint32_t acc, const uint4& v) {
  __half2 a = *reinterpret_cast<__half2*>(&acc);
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) a = __hmax2(a, __habs2(*reinterpret_cast<const __half2*>(&w[i])));
  return *reinterpret_cast<uint32_t*>(&a);
}
// The larger of the two packed maxima, widened.
template <typename T>
__device__ __forceinline__ float absmax_final(uint32_t acc) {
  const float2 f = T::widen2(acc);
  return fmaxf(f.x, f.y);
}

// ---- packed fp32 pairs (sm_100: one instruction, each lane rounded as the
// scalar op would be) ----

// Packed fp32 pairs: __fadd2_rn / __fmul2_rn / __ffma2_rn, one instruction
// per pair. A packed product that feeds a packed sum was observed to lose its
// own rounding on B200 (outputs one ulp off), with the intrinsic and with an
// inline PTX mul.rn.f32x2 alike, so every product that is then added is a
// scalar __fmul_rn (never contracted); packed multiplies only feed other
// multiplies or stores.
__device__ __forceinline__ float2 f2(float lo, float hi) { return make_float2(lo, hi); }

// acc[i] = acc[i] + w * m[i] for 8 values, product and sum each rounded once
// (scalar products, packed sums).
__device__ __forceinline__ void axpy8_rn(float (&acc)[8], float w, const float (&m)[8]) {
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    const float2 a =
        __fadd2_rn(f2(acc[i], acc[i + 1]), f2(__fmul_rn(w, m[i]), __fmul_rn(w, m[i + 1])));
    acc[i] = a.x;
    acc[i + 1] = a.y;
  }
}

// acc[i] = acc[i] + m[i] for 8 values.
__device__ __forceinline__ void add8_rn(float (&acc)[8], const float (&m)[8]) {
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    const float2 a = __fadd2_rn(f2(acc[i], acc[i + 1]), f2(m[i], m[i + 1]));
    acc[i] = a.x;
    acc[i + 1] = a.y;
  }
}

// ---- global memory access ----

// Read-only 16-byte load through the non-coherent path, not kept in L1.
__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Prefetch of the line holding p into L2 (no register is written; the later
// load finds the line there).
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__device__ __forceinline__ void st_v4(void* p, const uint4& v) {
  asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// ---- programmatic dependent launch (PDL) ----
// Every kernel lets its successor in the stream begin launching as soon as all
// of its CTAs are running, and waits for its predecessor's results (and their
// memory) before touching any data. Both are no-ops without the launch
// attribute.
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Integer rounding on the FMA pipe: for |r| <= 2^22, r + 1.5 * 2^23 lies in
// [2^23, 2^24), where fp32 values are spaced 1 apart, so the add itself rounds
// r to an integer n (round-to-nearest-even), and n sits in the low mantissa
// bits: for |n| <= 127 the low byte is n in two's complement.
constexpr float kRoundBias = 12582912.0f;        // 1.5 * 2^23
constexpr float kTieGuard = 0.49993896484375f;   // 0.5 - 2^-14

constexpr float kFastMinScale = 7.888609052210118e-31f;  // 2^-100

// The code of one value whose r = fl32(y * inv_scale) lies within 2^-14 of a
// half-integer h (n = rint(r), d = r - n), decided exactly without a division.
// Let Q = y / scale. D = y - h * scale is exact in fp32 (for 16-bit y and
// |Q - h| < 2^-13 it needs at most 11 significant bits), so one fma gives it.
// fl32(Q) equals h when |Q - h| is at most half the fp32 spacing on that side
// of h (h, with at most 9 significant bits, wins a tie at exactly half), i.e.
// when |D| <= spacing / 2 * scale (exact products of powers of two, no
// underflow for scale >= 2^-100); the spacing toward zero is halved at
// h = +-0.5, the only power of two among half-integers. The code is then the
// even one of h -+ 0.5 (round half to even), else the neighbour on Q's side.
__device__ __forceinline__ float tie_code_inline(float y, float scale, float n, float d) {
  const float h = n + (d > 0.0f ? 0.5f : -0.5f);
  const float D = __fmaf_rn(-h, scale, y);
  const float ah = fabsf(h);
  const float e = __uint_as_float(__float_as_uint(ah) & 0x7F800000u);  // 2^floor(log2|h|)
  const float u = e * 1.1920928955078125e-07f;                           // its spacing, 2^-23 e
  const bool away = D != 0.0f && ((D > 0.0f) == (h > 0.0f));
  const float lim = ((away || ah != e) ? u * 0.5f : u * 0.25f) * scale;
  const float lo = h - 0.5f, hi = h + 0.5f;
  const bool lo_even = (__float_as_uint(lo + kRoundBias) & 1u) == 0u;
  if (fabsf(D) <= lim) return lo_even ? lo : hi;
  return (away == (h > 0.0f)) ? hi : lo;
}

// The same decision as an out-of-line call: for kernels whose unrolled bodies
// would otherwise carry many inline copies of this rarely taken code.
static __device__ __noinline__ float tie_code_call(float y, float scale, float n, float d) {
  return tie_code_inline(y, scale, n, d);
}

// The int8 codes n[i] = rne(fl32(y[i] / scale)) of eight values, as fp32
// integers n and biased (b = n + 1.5 * 2^23, see above), for
// scale = fl32(max|row| / 127) > 0 and every |y[i]| <= max|row|. Then
// |y / scale| <= 127 (1 + 2^-23) and |n| <= 127, so no clamp is needed. With
// fast set (scale >= 2^-100, inv_scale = fl32(1 / scale)), r = y * inv_scale
// and the IEEE quotient fl32(y / scale) both lie within 127 * 3 * 2^-24 <
// 2^-15 of the exact quotient; when r is more than 2^-14 from every
// half-integer, both round to the same integer, and otherwise tie_code
// decides exactly (inline, or as a call with OUTLINE). Without fast (a tiny
// scale) the IEEE divisions decide.
template <bool OUTLINE = false>
__device__ __forceinline__ void quant_codes8(const float (&y)[8], float scale, float inv_scale,
                                             bool fast, float (&n)[8], float (&b)[8]) {
  if (fast) {
    const float2 bias2 = f2(kRoundBias, kRoundBias);
    const float2 nbias2 = f2(-kRoundBias, -kRoundBias);
    const float2 neg2 = f2(-1.0f, -1.0f);
    float d[8];
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      const float2 r2 = f2(__fmul_rn(y[i], inv_scale), __fmul_rn(y[i + 1], inv_scale));
      const float2 b2 = __fadd2_rn(r2, bias2);
      const float2 n2 = __fadd2_rn(b2, nbias2);
      const float2 d2 = __ffma2_rn(n2, neg2, r2);  // r - n, exact
      b[i] = b2.x;
      b[i + 1] = b2.y;
      n[i] = n2.x;
      n[i + 1] = n2.y;
      d[i] = d2.x;
      d[i + 1] = d2.y;
    }
    const float dmax =
        fmaxf(fmaxf(fmaxf(fabsf(d[0]), fabsf(d[1])), fmaxf(fabsf(d[2]), fabsf(d[3]))),
              fmaxf(fmaxf(fabsf(d[4]), fabsf(d[5])), fmaxf(fabsf(d[6]), fabsf(d[7]))));
    if (dmax >= kTieGuard) {  // one branch per vector, rarely taken
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (fabsf(d[i]) >= kTieGuard) {
          n[i] = OUTLINE ? tie_code_call(y[i], scale, n[i], d[i])
                         : tie_code_inline(y[i], scale, n[i], d[i]);
          b[i] = __fadd_rn(n[i], kRoundBias);
        }
    }
    return;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    b[i] = __fadd_rn(__fdiv_rn(y[i], scale), kRoundBias);
    n[i] = __fsub_rn(b[i], kRoundBias);
  }
}

// max |y[i]| over eight values, as a tree.
__device__ __forceinline__ float absmax8(const float (&y)[8]) {
  return fmaxf(fmaxf(fmaxf(fabsf(y[0]), fabsf(y[1])), fmaxf(fabsf(y[2]), fabsf(y[3]))),
               fmaxf(fmaxf(fabsf(y[4]), fabsf(y[5])), fmaxf(fabsf(y[6]), fabsf(y[7]))));
}

// Sixteen int8 codes of one row chunk as one 16-byte vector, element i in
// byte i; an all-zero row (amax == 0) gives zero codes.
__device__ __forceinline__ uint4 pack_codes16(const float (&y)[16], float amax, float scale,
                                              float inv_scale) {
  uint32_t w[4] = {0u, 0u, 0u, 0u};
  if (amax != 0.0f) {
    const bool fast = scale >= kFastMinScale;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float n[8], b[8];
      quant_codes8(reinterpret_cast<const float(&)[8]>(y[8 * h]), scale, inv_scale, fast, n, b);
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const uint32_t u0 = __float_as_uint(b[4 * k]), u1 = __float_as_uint(b[4 * k + 1]);
        const uint32_t u2 = __float_as_uint(b[4 * k + 2]), u3 = __float_as_uint(b[4 * k + 3]);
        w[2 * h + k] = __byte_perm(__byte_perm(u0, u1, 0x0040), __byte_perm(u2, u3, 0x0040), 0x5410);
      }
    }
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Eight int8 codes (element i in byte i) of one 16-byte vector of a row (the
// rare tie decisions as an out-of-line call with OUTLINE).
template <bool OUTLINE = false>
__device__ __forceinline__ uint2 pack_codes8(const float (&y)[8], float amax, float scale,
                                             float inv_scale) {
  if (amax == 0.0f) return make_uint2(0u, 0u);
  float n[8], b[8];
  quant_codes8<OUTLINE>(y, scale, inv_scale, scale >= kFastMinScale, n, b);
  uint32_t w[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const uint32_t u0 = __float_as_uint(b[4 * k]), u1 = __float_as_uint(b[4 * k + 1]);
    const uint32_t u2 = __float_as_uint(b[4 * k + 2]), u3 = __float_as_uint(b[4 * k + 3]);
    w[k] = __byte_perm(__byte_perm(u0, u1, 0x0040), __byte_perm(u2, u3, 0x0040), 0x5410);
  }
  return make_uint2(w[0], w[1]);
}

// m[i] = n[i] * scale, the fp32 values of the int8 round trip of eight values
// of a row (0 for an all-zero row), scale = fl32(amax / 127).
template <bool OUTLINE = false>
__device__ __forceinline__ void quant_roundtrip8(const float (&y)[8], float amax, float scale,
                                                 float inv_scale, float (&m)[8]) {
  if (amax == 0.0f) {
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = 0.0f;
    return;
  }
  float n[8], b[8];
  quant_codes8<OUTLINE>(y, scale, inv_scale, scale >= kFastMinScale, n, b);
  const float2 s2 = f2(scale, scale);
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    const float2 v = __fmul2_rn(f2(n[i], n[i + 1]), s2);
    m[i] = v.x;
    m[i + 1] = v.y;
  }
}

// Whether pair (t, k) is active under x_active_mask (1-D per token, 2-D per pair).
__device__ __forceinline__ bool pair_active(const uint8_t* mask, int mask_ndim, int t, int k,
                                            int K) {
  if (mask_ndim == 0) return true;
  if (mask_ndim == 1) return __ldg(mask + t) != 0;
  return __ldg(mask + static_cast<size_t>(t) * K + k) != 0;
}

// Resident blocks per SM of a kernel (occupancy API), cached per kernel and
// block size (a multiple of 32, at most 1024); each kernel is always launched
// with the same shared memory size.
template <auto Kernel>
int blocks_per_sm(int threads, size_t smem) {
  static int cached[33] = {};
  const int slot = threads >= 1024 ? 32 : threads / 32;
  if (cached[slot] == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, Kernel, threads, smem) != cudaSuccess ||
        n < 1)
      n = 1;
    cached[slot] = n;
  }
  return cached[slot];
}

}  // namespace moe
