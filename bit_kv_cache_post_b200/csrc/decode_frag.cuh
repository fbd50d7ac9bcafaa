// Register-level access to the packed cache for the tensor-core decode.
//
// The packed format (include/wushkv.h) is laid out so that the integer
// mma.sync fragments fall out of at most one shift and one mask per register:
//   * 2-bit K quads: word (ks, h, c) of a quad holds dims 32ks + 16h + 4c +
//     beta at byte beta for its four tokens at fields 0..3 -- masked to field
//     f it is the A fragment A[token 4 quad + f][k = 4c + 16h + beta] of
//     k-step ks (times 4^f), so m-tile f's fragments need no shift.
//   * 3- and 4-bit K rows: thread c of a quad of lanes (lane = 4r + c) reads
//     8 bytes per 2-bit plane of a token row; field ks of word (2c + h) holds
//     dims 32ks + 4c + 16h + beta at byte beta -- exactly the A fragment
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

// ---- fp16 mma.sync for the fp16 window tokens ------------------------------------
__device__ __forceinline__ void mma_f16_k16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                            uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16_k8(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm("mma.sync.aligned.m16n8k8.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(b0));
}

// Four 8x8 b16 matrices from shared memory; lane i supplies the address of
// row (i % 8) of matrix (i / 8).  Without .trans lane 4r + c receives
// (row r, cols 2c, 2c+1) of each matrix; with .trans (rows 2c, 2c+1, col r).
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&v)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&v)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
               : "r"(addr));
}

// ---- K rows -------------------------------------------------------------------
template <int BITS> struct KWords;   // 3- and 4-bit K rows
template <> struct KWords<3> { uint2 lo; uint32_t hi; };
template <> struct KWords<4> { uint4 w; };

// A fragment register of k-step ks, half h (k columns 16h + 4c .. +3).
template <int BITS>
__device__ __forceinline__ uint32_t k_frag(const KWords<BITS>& w, int ks, int h) {
  if constexpr (BITS == 3) {
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

// As v_frag, but masked in place (no shift): the codes come out multiplied
// by 2^(w * field).  For 2- and 4-bit planes the field of a PV row is fixed
// (rho = 2mt + rh), so every dim row carries one power-of-two factor that is
// removed once from the final output (v_row_scale).
template <int BITS>
__device__ __forceinline__ uint32_t v_frag_scaled(const VWords<BITS>& v, int rho) {
  static_assert(BITS == 2 || BITS == 4, "shift-free fragments need a single plane");
  if constexpr (BITS == 2) {
    return pick4(v.lo, rho >> 2) & (0x03030303u << (2 * (rho & 3)));
  } else {
    const uint32_t word = (rho >> 1) < 4 ? pick4(v.a, rho >> 1) : pick4(v.b, (rho >> 1) - 4);
    return word & (0x0F0F0F0Fu << (4 * (rho & 1)));
  }
}

// 1 / (factor of v_frag_scaled) for rho.
template <int BITS>
__device__ __forceinline__ float v_row_scale(int rho) {
  if constexpr (BITS == 2) return 1.f / (float)(1 << (2 * (rho & 3)));
  else return (rho & 1) ? 1.f / 16.f : 1.f;
}

}  // namespace wushkv
