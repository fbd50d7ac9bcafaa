// Register-level access to the packed cache for the tensor-core decode.
//
// The packed format (include/wushkv.h) is laid out so that the integer
// mma.sync fragments fall out of one shift and one mask per register:
//   * K rows: thread c of a quad of lanes (lane = 4r + c) reads 8 bytes per
//     2-bit plane of a token row; field ks of word (2c + h) holds dims
//     32ks + 4c + 16h + beta at byte beta -- exactly the A fragment
//     A[token][k = 4c + 16h + beta] of k-step ks of an m16n8k32 product.
//   * V quads: word (r, j) field s holds dim 16mt + r + 8rh (rho = 2mt + rh)
//     of the quad's 4 tokens at bytes 0..3 -- the A fragment
//     A[dim][k = 4 consecutive tokens] of the transposed PV product.
#pragma once

#include "wushkv_internal.cuh"

namespace wushkv {

// ---- integer mma.sync (m16n8k32, s32 accumulate) -----------------------------
__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_u8u8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ---- K rows -------------------------------------------------------------------
template <int BITS> struct KWords;
template <> struct KWords<2> { uint2 lo; };
template <> struct KWords<3> { uint2 lo; uint32_t hi; };
template <> struct KWords<4> { uint4 w; };

template <int BITS>
__device__ __forceinline__ KWords<BITS> load_k_words(const uint8_t* p0, const uint8_t* p1, int tok,
                                                     int c4) {
  KWords<BITS> r;
  if constexpr (BITS == 2) {
    r.lo = __ldg(reinterpret_cast<const uint2*>(p0 + (size_t)tok * 32) + c4);
  } else if constexpr (BITS == 3) {
    r.lo = __ldg(reinterpret_cast<const uint2*>(p0 + (size_t)tok * 32) + c4);
    r.hi = __ldg(reinterpret_cast<const uint32_t*>(p1 + (size_t)tok * 16) + c4);
  } else {
    r.w = __ldg(reinterpret_cast<const uint4*>(p0 + (size_t)tok * 64) + c4);
  }
  return r;
}

// A fragment register of k-step ks, half h (k columns 16h + 4c .. +3).
template <int BITS>
__device__ __forceinline__ uint32_t k_frag(const KWords<BITS>& w, int ks, int h) {
  if constexpr (BITS == 2) {
    return ((h ? w.lo.y : w.lo.x) >> (2 * ks)) & 0x03030303u;
  } else if constexpr (BITS == 3) {
    const uint32_t lo = ((h ? w.lo.y : w.lo.x) >> (2 * ks)) & 0x03030303u;
    const int rho = 4 * h + ks;
    return lo | (((w.hi >> rho) & 0x01010101u) << 2);
  } else {
    const int j = 2 * h + (ks >> 1);
    const uint32_t word = j == 0 ? w.w.x : j == 1 ? w.w.y : j == 2 ? w.w.z : w.w.w;
    return (word >> (4 * (ks & 1))) & 0x0F0F0F0Fu;
  }
}

// ---- V quads ------------------------------------------------------------------
template <int BITS> struct VWords;
template <> struct VWords<2> { uint4 lo; };
template <> struct VWords<3> { uint4 lo; uint2 hi; };
template <> struct VWords<4> { uint4 a, b; };

template <int BITS>
__device__ __forceinline__ VWords<BITS> load_v_words(const uint8_t* p0, const uint8_t* p1, int quad,
                                                     int r) {
  VWords<BITS> v;
  if constexpr (BITS == 2) {
    v.lo = __ldg(reinterpret_cast<const uint4*>(p0 + (size_t)quad * 128) + r);
  } else if constexpr (BITS == 3) {
    v.lo = __ldg(reinterpret_cast<const uint4*>(p0 + (size_t)quad * 128) + r);
    v.hi = __ldg(reinterpret_cast<const uint2*>(p1 + (size_t)quad * 64) + r);
  } else {
    const uint4* q = reinterpret_cast<const uint4*>(p0 + (size_t)quad * 256) + 2 * r;
    v.a = __ldg(q);
    v.b = __ldg(q + 1);
  }
  return v;
}

__device__ __forceinline__ uint32_t pick4(const uint4& w, int j) {
  return j == 0 ? w.x : j == 1 ? w.y : j == 2 ? w.z : w.w;
}

// A fragment register for rho = 2mt + rh: dim 16mt + r + 8rh, 4 tokens.
template <int BITS>
__device__ __forceinline__ uint32_t v_frag(const VWords<BITS>& v, int rho) {
  if constexpr (BITS == 2) {
    return (pick4(v.lo, rho >> 2) >> (2 * (rho & 3))) & 0x03030303u;
  } else if constexpr (BITS == 3) {
    const uint32_t lo = (pick4(v.lo, rho >> 2) >> (2 * (rho & 3))) & 0x03030303u;
    const uint32_t hw = (rho >> 3) ? v.hi.y : v.hi.x;
    return lo | (((hw >> (rho & 7)) & 0x01010101u) << 2);
  } else {
    const uint32_t word = (rho >> 1) < 4 ? pick4(v.a, rho >> 1) : pick4(v.b, (rho >> 1) - 4);
    return (word >> (4 * (rho & 1))) & 0x0F0F0F0Fu;
  }
}

// Per-token dequantisation parameters: value = scale * code + offset.
template <bool AFFINE>
__device__ __forceinline__ float2 load_meta(const uint8_t* meta, int tok, float beta) {
  if constexpr (AFFINE) {
    const __half2 sl = *reinterpret_cast<const __half2*>(meta + (size_t)tok * 4);
    return make_float2(__low2float(sl), __high2float(sl));
  } else {
    const float d = __half2float(*reinterpret_cast<const __half*>(meta + (size_t)tok * 2));
    return make_float2(d, d * beta);
  }
}

}  // namespace wushkv
