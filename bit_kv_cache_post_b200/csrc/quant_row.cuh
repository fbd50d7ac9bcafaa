// One thread per token vector: per-token quantiser parameters, codes and
// packed words for the bulk-append kernels.
//
// Method source: summary page "WUSH-KV：数据自适应变换的 KV Cache 低比特量化"
// (ai-papers-daily), section 方法关键点 (per-token QuEST INT quantiser with an
// RMS-based step and bin-centre reconstruction; OSCAR-style percentile-clipped
// affine quantiser).  Every step below is the exact fp32 arithmetic of the
// FMA append kernel's warp quantisers, reorganised for one thread per vector:
//   QuEST:  Delta = fp16(alpha * sqrt(sum x^2 / 128) / 2^(b-1)), sum in float64;
//           inv = RN(1 / Delta) (0 for Delta = 0);
//           code = clamp(floor(RN(RN(x * inv) + L/2)), 0, L-1)
//   affine: lo, hi = order statistics r_lo, r_hi (r_lo in {1,2}, r_hi in
//           {127,128}); s = fp16(RN(RN(hi - lo) / (L-1))); inv = RN(1 / s);
//           code = clamp(rint(RN(RN(x - lo) * inv)), 0, L-1)
// x is always the fp16 value of the element.  Codes are produced as the bit
// pattern of (clamped t) + 1.5 * 2^23, whose low byte is the code and whose
// second byte is zero.
#pragma once

#include "wushkv_internal.cuh"

namespace wushkv {
namespace rowq {

constexpr uint32_t MAGIC = 0x4B400000u;   // bit pattern of 1.5 * 2^23

// Sum of 2^bit over the fields of a fully populated packed word of width w.
__host__ __device__ constexpr uint32_t field_bit_sum(int w) {
  uint32_t s = 0;
  for (int f = 0; f < 8 / w; ++f) s += 1u << (w * f);
  return s * 0x01010101u;
}

__device__ __forceinline__ __half2 bf16x2_to_h2(uint32_t u) {
  return __floats2half2_rn(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}

__device__ __forceinline__ __half2 f32x2_to_h2(uint32_t a, uint32_t b) {
  return __floats2half2_rn(__uint_as_float(a), __uint_as_float(b));
}

// ---- per-token statistics ----------------------------------------------------------

// Two smallest and two largest values per half lane, fed two half2 at a
// time: the pair is ordered first, then merged into each sorted pair with
//   second = min(max(a1, mn), min(a2, mx)),  first = min(a1, mn).
struct AffineStats {
  __half2 a1, a2, b1, b2;
  __device__ __forceinline__ void init() {
    a1 = a2 = __half2half2(__ushort_as_half((unsigned short)0x7C00u));   // +inf
    b1 = b2 = __half2half2(__ushort_as_half((unsigned short)0xFC00u));   // -inf
  }
  __device__ __forceinline__ void add2(__half2 x, __half2 y) {
    const __half2 mn = __hmin2(x, y), mx = __hmax2(x, y);
    a2 = __hmin2(__hmin2(a2, mx), __hmax2(a1, mn));
    a1 = __hmin2(a1, mn);
    b2 = __hmax2(__hmax2(b2, mn), __hmin2(b1, mx));
    b1 = __hmax2(b1, mx);
  }
};

struct QParams {
  float2 neglo;    // affine: (-lo, -lo)
  __half2 lo2;     // affine: (lo, lo)
  float2 inv;      // (inv, inv)
  uint32_t meta;   // QuEST: Delta (fp16 bits); affine: s | lo << 16
};

__device__ __forceinline__ void affine_finish(const AffineStats& st, int bits, bool lo_second,
                                              bool hi_second, QParams& q) {
  const float a1l = __low2float(st.a1), a1h = __high2float(st.a1);
  const float a2l = __low2float(st.a2), a2h = __high2float(st.a2);
  const float b1l = __low2float(st.b1), b1h = __high2float(st.b1);
  const float b2l = __low2float(st.b2), b2h = __high2float(st.b2);
  float lo = lo_second ? fminf(fmaxf(a1l, a1h), fminf(a2l, a2h)) : fminf(a1l, a1h);
  float hi = hi_second ? fmaxf(fminf(b1l, b1h), fmaxf(b2l, b2h)) : fmaxf(b1l, b1h);
  lo = __fadd_rn(lo, 0.f);   // -0 -> +0
  hi = __fadd_rn(hi, 0.f);
  const __half lo_h = __float2half_rn(lo);
  const __half s_h = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), (float)((1 << bits) - 1)));
  const float sd = __half2float(s_h), lof = __half2float(lo_h);
  const float inv = (sd == 0.f) ? 0.f : __frcp_rn(sd);
  q.neglo = make_float2(-lof, -lof);
  q.lo2 = __half2half2(lo_h);
  q.inv = make_float2(inv, inv);
  q.meta = (uint32_t)__half_as_ushort(s_h) | ((uint32_t)__half_as_ushort(lo_h) << 16);
}

struct QuestStats {
  double ss0, ss1;
  __device__ __forceinline__ void init() { ss0 = ss1 = 0.0; }
  __device__ __forceinline__ void add(__half2 x) {
    const float2 f = __half22float2(x);
    ss0 = __fma_rn((double)f.x, (double)f.x, ss0);
    ss1 = __fma_rn((double)f.y, (double)f.y, ss1);
  }
};

__device__ __forceinline__ void quest_finish(const QuestStats& st, int bits, double alpha,
                                             QParams& q) {
  const double rms = __dsqrt_rn((st.ss0 + st.ss1) / 128.0);
  const __half dl = f64_to_f16_rn(__dmul_rn(alpha, rms) / (double)(1 << (bits - 1)));
  const float d32 = __half2float(dl);
  const float inv = (d32 == 0.f) ? 0.f : __frcp_rn(d32);
  q.neglo = make_float2(0.f, 0.f);
  q.lo2 = __float2half2_rn(0.f);
  q.inv = make_float2(inv, inv);
  q.meta = __half_as_ushort(dl);
}

// ---- codes ------------------------------------------------------------------------------

// Packed fp32 arithmetic (two lanes per instruction) with an explicit
// rounding mode.  Only for steps that cannot be contracted into a fused
// multiply-add: on sm_100 a packed multiply feeding a packed add was
// observed to fuse even with explicit .rn (rounding the product only once),
// so a packed multiply is always followed by a clamp before any add, and the
// QuEST step x * inv + L/2 uses the scalar intrinsics, which never contract.
__device__ __forceinline__ float2 mul2_rn(float2 a, float2 b) {
  float2 r;
  asm("{\n .reg .b64 a, b, d;\n mov.b64 a, {%2, %3};\n mov.b64 b, {%4, %5};\n"
      " mul.rn.f32x2 d, a, b;\n mov.b64 {%0, %1}, d;\n}\n"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}
__device__ __forceinline__ float2 add2_rn(float2 a, float2 b) {
  float2 r;
  asm("{\n .reg .b64 a, b, d;\n mov.b64 a, {%2, %3};\n mov.b64 b, {%4, %5};\n"
      " add.rn.f32x2 d, a, b;\n mov.b64 {%0, %1}, d;\n}\n"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}
__device__ __forceinline__ float2 add2_rm(float2 a, float2 b) {
  float2 r;
  asm("{\n .reg .b64 a, b, d;\n mov.b64 a, {%2, %3};\n mov.b64 b, {%4, %5};\n"
      " add.rm.f32x2 d, a, b;\n mov.b64 {%0, %1}, d;\n}\n"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}

// Code patterns (MAGIC + code) of the two elements of x2.
template <bool AFFINE, int L>
__device__ __forceinline__ uint2 code_pat2(__half2 x2, const QParams& q) {
  const float2 magic = make_float2(12582912.f, 12582912.f);
  float2 t;
  if constexpr (AFFINE) {
    // raising x to lo keeps t >= 0: only the upper clamp remains
    t = mul2_rn(add2_rn(__half22float2(__hmax2(x2, q.lo2)), q.neglo), q.inv);
    t.x = fminf(t.x, (float)(L - 1));
    t.y = fminf(t.y, (float)(L - 1));
    t = add2_rn(t, magic);                 // rint, ties to even
  } else {
    const float2 f = __half22float2(x2);
    t.x = __fadd_rn(__fmul_rn(f.x, q.inv.x), (float)(L / 2));
    t.y = __fadd_rn(__fmul_rn(f.y, q.inv.y), (float)(L / 2));
    t.x = fminf(fmaxf(t.x, 0.f), (float)(L - 1));
    t.y = fminf(fmaxf(t.y, 0.f), (float)(L - 1));
    t = add2_rm(t, magic);                 // floor
  }
  return make_uint2(__float_as_uint(t.x), __float_as_uint(t.y));
}

// ---- V quads ----------------------------------------------------------------------------

// 4x4 byte transpose among the four lanes of a quad (lanes spaced STRIDE
// apart, quad index b): lane b' receives, in byte b, byte b' of lane b's x.
template <int STRIDE>
__device__ __forceinline__ uint32_t quad_transpose(uint32_t x, uint32_t sel_a, uint32_t sel_b) {
  const uint32_t r = __shfl_xor_sync(FULL, x, 2 * STRIDE);
  const uint32_t z = __byte_perm(x, r, sel_a);
  const uint32_t w = __shfl_xor_sync(FULL, z, STRIDE);
  return __byte_perm(z, w, sel_b);
}
__device__ __forceinline__ void quad_selectors(int b, uint32_t& sel_a, uint32_t& sel_b) {
  sel_a = (b & 2) ? 0x3276u : 0x5410u;   // keep bytes 2,3 / 0,1 of own word
  sel_b = (b & 1) ? 0x3715u : 0x6240u;   // odd / even bytes
}

// V quad of 4 tokens (packed format of wushkv.h): word (r, j) of a plane of
// width w holds, in byte beta, the codes of token beta for dims
// 16 mt + r + 8 rh (rho = 2 mt + rh, j = rho / (8/w), field rho mod (8/w)).
// Each lane builds, for k in {0, 1} and every j, the word whose byte b is
// its own contribution to word (2b + k, j); the quad transpose then leaves
// lane b with the complete words of row units 2b and 2b + 1, stored at their
// rotated unit positions (r + 2 (quad mod 4)) mod 8 (4-bit units split into
// two 16-byte halves 128 bytes apart).  Every lane of the warp must call.
template <int BITS, bool AFFINE, int STRIDE>
__device__ __forceinline__ void emit_v_quad(const __half2 (&xh)[64], const QParams& q, int beta,
                                            int quad, uint8_t* quad0, uint8_t* quad1, bool valid) {
  constexpr int L = 1 << BITS;
  constexpr int W0 = BITS == 3 ? 2 : BITS;
  constexpr int P0 = 8 / W0;
  uint32_t x0[2][2 * W0], x1[2][2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
#pragma unroll
    for (int j = 0; j < 2 * W0; ++j) x0[k][j] = 0u;
    x1[k][0] = x1[k][1] = 0u;
  }
  // element pairs (d, d + 1), d even, have r and r + 1: words k = 0 and 1
#pragma unroll
  for (int e = 0; e < 64; ++e) {
    const int d = 2 * e;
    const int r = d & 7, rh = (d >> 3) & 1, mt = d >> 4;
    const int rho = 2 * mt + rh, bb = r >> 1;
    const uint2 p = code_pat2<AFFINE, L>(xh[e], q);
    if constexpr (BITS == 3) {
      x0[0][rho >> 2] += (p.x & 3u) << (8 * bb + 2 * (rho & 3));
      x0[1][rho >> 2] += (p.y & 3u) << (8 * bb + 2 * (rho & 3));
      x1[0][rho >> 3] += ((p.x >> 2) & 1u) << (8 * bb + (rho & 7));
      x1[1][rho >> 3] += ((p.y >> 2) & 1u) << (8 * bb + (rho & 7));
    } else {
      x0[0][rho / P0] += p.x << (8 * bb + W0 * (rho % P0));
      x0[1][rho / P0] += p.y << (8 * bb + W0 * (rho % P0));
    }
  }
  if constexpr (BITS != 3) {
    constexpr uint32_t corr = MAGIC * field_bit_sum(W0);
#pragma unroll
    for (int k = 0; k < 2; ++k)
#pragma unroll
      for (int j = 0; j < 2 * W0; ++j) x0[k][j] -= corr;
  }
  uint32_t sa, sb;
  quad_selectors(beta, sa, sb);
#pragma unroll
  for (int k = 0; k < 2; ++k) {
#pragma unroll
    for (int j = 0; j < 2 * W0; ++j) x0[k][j] = quad_transpose<STRIDE>(x0[k][j], sa, sb);
    if constexpr (BITS == 3) {
      x1[k][0] = quad_transpose<STRIDE>(x1[k][0], sa, sb);
      x1[k][1] = quad_transpose<STRIDE>(x1[k][1], sa, sb);
    }
  }
  if (!valid) return;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int pos = (2 * beta + k + 2 * (quad & 3)) & 7;
    *reinterpret_cast<uint4*>(quad0 + 16 * pos) = make_uint4(x0[k][0], x0[k][1], x0[k][2], x0[k][3]);
    if constexpr (W0 == 4)
      *reinterpret_cast<uint4*>(quad0 + 128 + 16 * pos) =
          make_uint4(x0[k][4], x0[k][5], x0[k][6], x0[k][7]);
    if constexpr (BITS == 3)
      *reinterpret_cast<uint2*>(quad1 + 8 * pos) = make_uint2(x1[k][0], x1[k][1]);
  }
}

// As emit_v_quad, for a lane holding one half of the token's dims (half hf:
// dims 64 hf .. 64 hf + 63 in xh[0..31]).  Its dims carry rho in
// [8 hf, 8 hf + 8), i.e. the words j in [hf 8/(8/w), (hf + 1) 8/(8/w)) of
// every row unit; the quad transpose runs among the lanes of the same half
// (STRIDE apart).  Every lane of the warp must call.
template <int BITS, bool AFFINE, int STRIDE>
__device__ __forceinline__ void emit_v_quad_half(const __half2 (&xh)[32], const QParams& q, int beta,
                                                 int hf, int quad, uint8_t* quad0, uint8_t* quad1,
                                                 bool valid) {
  constexpr int L = 1 << BITS;
  constexpr int W0 = BITS == 3 ? 2 : BITS;
  constexpr int P0 = 8 / W0;
  constexpr int NJ = 8 / P0;                // words of the half per row unit (= w)
  uint32_t x0[2][NJ], x1[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
#pragma unroll
    for (int j = 0; j < NJ; ++j) x0[k][j] = 0u;
    x1[k] = 0u;
  }
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    const int dl = 2 * e;                   // dim within the half (d = 64 hf + dl)
    const int r = dl & 7, rh = (dl >> 3) & 1;
    const int rl = 2 * (dl >> 4) + rh;      // rho - 8 hf
    const int bb = r >> 1;
    const uint2 p = code_pat2<AFFINE, L>(xh[e], q);
    if constexpr (BITS == 3) {
      x0[0][rl >> 2] += (p.x & 3u) << (8 * bb + 2 * (rl & 3));
      x0[1][rl >> 2] += (p.y & 3u) << (8 * bb + 2 * (rl & 3));
      x1[0] += ((p.x >> 2) & 1u) << (8 * bb + rl);
      x1[1] += ((p.y >> 2) & 1u) << (8 * bb + rl);
    } else {
      x0[0][rl / P0] += p.x << (8 * bb + W0 * (rl % P0));
      x0[1][rl / P0] += p.y << (8 * bb + W0 * (rl % P0));
    }
  }
  if constexpr (BITS != 3) {
    constexpr uint32_t corr = MAGIC * field_bit_sum(W0);
#pragma unroll
    for (int k = 0; k < 2; ++k)
#pragma unroll
      for (int j = 0; j < NJ; ++j) x0[k][j] -= corr;
  }
  uint32_t sa, sb;
  quad_selectors(beta, sa, sb);
#pragma unroll
  for (int k = 0; k < 2; ++k) {
#pragma unroll
    for (int j = 0; j < NJ; ++j) x0[k][j] = quad_transpose<STRIDE>(x0[k][j], sa, sb);
    if constexpr (BITS == 3) x1[k] = quad_transpose<STRIDE>(x1[k], sa, sb);
  }
  if (!valid) return;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int pos = (2 * beta + k + 2 * (quad & 3)) & 7;
    if constexpr (W0 == 2) {
      *reinterpret_cast<uint2*>(quad0 + 16 * pos + 8 * hf) = make_uint2(x0[k][0], x0[k][1]);
    } else {
      *reinterpret_cast<uint4*>(quad0 + 128 * hf + 16 * pos) =
          make_uint4(x0[k][0], x0[k][1], x0[k][2], x0[k][3]);
    }
    if constexpr (BITS == 3) *reinterpret_cast<uint32_t*>(quad1 + 8 * pos + 4 * hf) = x1[k];
  }
}

// Merge the statistics of the two halves of a token (lanes `lane ^ 1`).
__device__ __forceinline__ void affine_merge_pair(AffineStats& st) {
  auto xch = [](__half2 v) {
    const uint32_t u = __shfl_xor_sync(FULL, *reinterpret_cast<const uint32_t*>(&v), 1);
    return *reinterpret_cast<const __half2*>(&u);
  };
  const __half2 a1 = xch(st.a1), a2 = xch(st.a2), b1 = xch(st.b1), b2 = xch(st.b2);
  st.a2 = __hmin2(__hmax2(st.a1, a1), __hmin2(st.a2, a2));
  st.a1 = __hmin2(st.a1, a1);
  st.b2 = __hmax2(__hmin2(st.b1, b1), __hmax2(st.b2, b2));
  st.b1 = __hmax2(st.b1, b1);
}
__device__ __forceinline__ void quest_merge_pair(QuestStats& st) {
  const double s = st.ss0 + st.ss1;
  const double o = __shfl_xor_sync(FULL, s, 1);
  st.ss0 = s;
  st.ss1 = o;
}

}  // namespace rowq
}  // namespace wushkv
