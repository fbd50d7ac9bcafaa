// Bulk (prefill) append on the fifth-generation tensor cores.
//
// Method source: summary page "WUSH-KV：数据自适应变换的 KV Cache 低比特量化"
// (ai-papers-daily), sections 工作参考价值 and 方法关键点: keys are multiplied by
// the per-head transform after RoPE (K' = K T^T for a block of tokens), values
// pass through unchanged, and every token vector that leaves the fp16 recent
// window is quantised per token (QuEST INT or percentile-clipped affine) and
// bit-packed.  This kernel handles the tokens of one append that go straight
// from the input to the packed cache; the window rows, the flush of old ring
// rows and a partial first quad stay with the FMA append kernel.
//
// Design (one CTA per SM, 12 warps, all tiles of a CTA from one KV head):
//   warp 0      TMA producer: 128-token K and V tiles (bf16, 128-byte swizzle)
//               through a two-stage ring each;
//   warp 1      tensor-memory owner and MMA issuer: K' = K T_lo^T + K T_mid^T
//               + K T_hi^T with T = T_hi + T_mid + T_lo split into three bf16
//               matrices (T to about 2^-27 relative, so K' is as close to the
//               exact product as an fp32 FMA loop), fp32 accumulation in
//               TMEM, two 128-column accumulators;
//   warps 4-7, 8-11  two epilogue warpgroups taking alternate tiles; thread
//               i owns token row i: K' from TMEM lane i and V from the
//               swizzled smem tile, rounded to fp16 into 64 half2 registers,
//               then per-token statistics, codes, and packed stores (the V
//               quad words assembled by byte transposes among the quad's
//               four lanes).
// Every wait is bounded; on a timeout the CTA records DEV_ERR_TIMEOUT, stops
// issuing, waits (bounded) for its own copies and MMAs, frees TMEM and ends.
#include <cuda.h>

#include "wushkv_internal.cuh"
#include "tcgen05.cuh"

namespace wushkv {

namespace {

constexpr int TILE = 128;                    // tokens per tile (MMA M)
constexpr int NTHREADS = 384;
constexpr int TILE_BYTES = TILE * D * 2;     // one bf16 tile, 32 KB
constexpr int HALF_BYTES = TILE_BYTES / 2;   // 64 dims (one 128-byte swizzle span)
constexpr uint32_t PF_WAIT_POLLS = 1u << 22;

// shared memory map (offsets from a 1024-byte aligned base)
constexpr int OFF_THI = 0;
constexpr int OFF_TMID = OFF_THI + TILE_BYTES;
constexpr int OFF_TLO = OFF_TMID + TILE_BYTES;
constexpr int OFF_K = OFF_TLO + TILE_BYTES;           // 2 stages
constexpr int OFF_V = OFF_K + 2 * TILE_BYTES;         // 2 stages
constexpr int OFF_BAR = OFF_V + 2 * TILE_BYTES;
constexpr int N_BARS = 13;
constexpr int OFF_MISC = OFF_BAR + 8 * N_BARS;
constexpr int SMEM_USED = OFF_MISC + 16;
constexpr int SMEM_BYTES = SMEM_USED + 1024;          // slack for the alignment
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");

// bit pattern of 1.5 * 2^23: adding it to t in [-2^22, 2^22] leaves the
// rounded integer in the low mantissa bits
constexpr int MAGIC = 0x4B400000;

// Sum over the fields of a fully populated packed word of 2^bit: every word
// of a plane of width w holds 8/w fields in each of its 4 bytes.
__host__ __device__ constexpr uint32_t field_bit_sum(int w) {
  uint32_t s = 0;
  for (int f = 0; f < 8 / w; ++f) s += 1u << (w * f);
  return s * 0x01010101u;
}

__device__ __forceinline__ __half2 bf16x2_to_h2(uint32_t u) {
  return __floats2half2_rn(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}

// MAGIC + code of one element (exact fp32 steps of the quantiser).
//   QuEST:  t = RN(RN(x * inv) + L/2), code = clamp(floor(t), 0, L-1)
//   affine: t = RN(RN(x - lo) * inv), code = clamp(rint(t), 0, L-1); the
//           caller has already raised x to lo, so t >= 0.
// inv is 0 for a zero step (QuEST: every code L/2; affine: every code 0).
template <bool AFFINE, int L>
__device__ __forceinline__ int code_pat(float x, float lo, float inv) {
  if constexpr (AFFINE) {
    const float t = __fmul_rn(__fsub_rn(x, lo), inv);
    return min(__float_as_int(__fadd_rn(t, 12582912.f)), MAGIC + L - 1);
  } else {
    const float t = __fadd_rn(__fmul_rn(x, inv), (float)(L / 2));
    return min(max(__float_as_int(__fadd_rd(t, 12582912.f)), MAGIC), MAGIC + L - 1);
  }
}

// Per-token parameters of the QuEST quantiser: Delta = alpha * RMS / 2^(b-1)
// with the sum of squares in float64 and Delta rounded once to fp16.
__device__ __forceinline__ void quest_params(const __half2 (&xh)[64], int bits, double alpha,
                                             float& inv, uint32_t& meta) {
  double ss[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
  for (int e = 0; e < 64; ++e) {
    const float2 f = __half22float2(xh[e]);
    ss[e & 3] = __fma_rn((double)f.x, (double)f.x, ss[e & 3]);
    ss[e & 3] = __fma_rn((double)f.y, (double)f.y, ss[e & 3]);
  }
  const double sum = (ss[0] + ss[1]) + (ss[2] + ss[3]);
  const double rms = __dsqrt_rn(sum / 128.0);
  const double dd = __dmul_rn(alpha, rms) / (double)(1 << (bits - 1));
  const __half dl = f64_to_f16_rn(dd);
  const float d32 = __half2float(dl);
  inv = (d32 == 0.f) ? 0.f : __frcp_rn(d32);
  meta = __half_as_ushort(dl);
}

// Per-token parameters of the percentile-clipped affine quantiser with
// r_lo in {1, 2} and r_hi in {127, 128}: the two smallest and two largest
// values are tracked per half lane, then the lanes are merged.
__device__ __forceinline__ void affine_params(const __half2 (&xh)[64], int bits, bool lo_second,
                                              bool hi_second, float& lo_f, float& inv,
                                              uint32_t& meta) {
  const __half2 pinf = __half2half2(__ushort_as_half((unsigned short)0x7C00u));
  const __half2 ninf = __half2half2(__ushort_as_half((unsigned short)0xFC00u));
  __half2 a1 = pinf, a2 = pinf, b1 = ninf, b2 = ninf;
#pragma unroll
  for (int e = 0; e < 64; ++e) {
    const __half2 x = xh[e];
    a2 = __hmin2(a2, __hmax2(a1, x));
    a1 = __hmin2(a1, x);
    b2 = __hmax2(b2, __hmin2(b1, x));
    b1 = __hmax2(b1, x);
  }
  const float a1l = __low2float(a1), a1h = __high2float(a1);
  const float a2l = __low2float(a2), a2h = __high2float(a2);
  const float b1l = __low2float(b1), b1h = __high2float(b1);
  const float b2l = __low2float(b2), b2h = __high2float(b2);
  float lo = lo_second ? fminf(fmaxf(a1l, a1h), fminf(a2l, a2h)) : fminf(a1l, a1h);
  float hi = hi_second ? fmaxf(fminf(b1l, b1h), fmaxf(b2l, b2h)) : fmaxf(b1l, b1h);
  lo = __fadd_rn(lo, 0.f);   // -0 -> +0
  hi = __fadd_rn(hi, 0.f);
  const __half lo_h = __float2half_rn(lo);
  const float s32 = __fdiv_rn(__fsub_rn(hi, lo), (float)((1 << bits) - 1));
  const __half s_h = __float2half_rn(s32);
  const float sd = __half2float(s_h);
  lo_f = __half2float(lo_h);
  inv = (sd == 0.f) ? 0.f : __frcp_rn(sd);
  meta = (uint32_t)__half_as_ushort(s_h) | ((uint32_t)__half_as_ushort(lo_h) << 16);
}

// K row of one token (packed format of wushkv.h): dim d = 32 ks + 4 c + 16 h
// + beta goes to word c w + rho / (8/w), field rho mod (8/w), byte beta,
// with rho = 4 h + ks.
template <int BITS, bool AFFINE>
__device__ __forceinline__ void emit_k_row(const __half2 (&xh)[64], float lo, float inv,
                                           uint8_t* row0, uint8_t* row1) {
  constexpr int L = 1 << BITS;
  constexpr int W0 = BITS == 3 ? 2 : BITS;
  constexpr int NW0 = 4 * W0;
  uint32_t w0[NW0], w1[4];
#pragma unroll
  for (int i = 0; i < NW0; ++i) w0[i] = 0u;
#pragma unroll
  for (int i = 0; i < 4; ++i) w1[i] = 0u;
  const __half2 lo2 = __float2half2_rn(lo);
#pragma unroll
  for (int d = 0; d < D; ++d) {
    const int ks = d >> 5, c = (d >> 2) & 3, h = (d >> 4) & 1, beta = d & 3;
    const int rho = 4 * h + ks;
    const __half2 x2 = AFFINE ? __hmax2(xh[d >> 1], lo2) : xh[d >> 1];
    const float x = (d & 1) ? __high2float(x2) : __low2float(x2);
    const int p = code_pat<AFFINE, L>(x, lo, inv);
    if constexpr (BITS == 3) {
      w0[2 * c + (rho >> 2)] += (uint32_t)(p & 3) << (8 * beta + 2 * (rho & 3));
      w1[c] += (uint32_t)((p >> 2) & 1) << (8 * beta + rho);
    } else {
      constexpr int P = 8 / W0;
      w0[c * W0 + rho / P] += (uint32_t)p << (8 * beta + W0 * (rho % P));
    }
  }
  if constexpr (BITS != 3) {
    constexpr uint32_t corr = (uint32_t)MAGIC * field_bit_sum(W0);
#pragma unroll
    for (int i = 0; i < NW0; ++i) w0[i] -= corr;
  }
  uint4* o0 = reinterpret_cast<uint4*>(row0);
#pragma unroll
  for (int i = 0; i < NW0 / 4; ++i)
    o0[i] = make_uint4(w0[4 * i], w0[4 * i + 1], w0[4 * i + 2], w0[4 * i + 3]);
  if constexpr (BITS == 3) *reinterpret_cast<uint4*>(row1) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
}

// 4x4 byte transpose among the four lanes of a quad (lanes 4q .. 4q+3,
// lane index b = lane % 4): lane b' receives, in byte b, byte b' of lane
// b's x.  Two exchanges: 16-bit halves with lane b^2, then bytes with b^1.
// sel_a / sel_b: the lane's byte-permute selectors (quad_selectors).
__device__ __forceinline__ uint32_t quad_transpose(uint32_t x, uint32_t sel_a, uint32_t sel_b) {
  const uint32_t r = __shfl_xor_sync(FULL, x, 2);
  const uint32_t z = __byte_perm(x, r, sel_a);
  const uint32_t w = __shfl_xor_sync(FULL, z, 1);
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
// lane b with the complete words of row units 2b and 2b + 1, which it
// stores at their rotated unit positions (r + 2 (quad mod 4)) mod 8 (4-bit
// units split into two 16-byte halves 128 bytes apart).
template <int BITS, bool AFFINE>
__device__ __forceinline__ void emit_v_quad(const __half2 (&xh)[64], float lo, float inv, int beta,
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
  const __half2 lo2 = __float2half2_rn(lo);
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int k = r & 1, bb = r >> 1;
#pragma unroll
    for (int rho = 0; rho < 16; ++rho) {
      const int d = 16 * (rho >> 1) + r + 8 * (rho & 1);
      const __half2 x2 = AFFINE ? __hmax2(xh[d >> 1], lo2) : xh[d >> 1];
      const float x = (d & 1) ? __high2float(x2) : __low2float(x2);
      const int p = code_pat<AFFINE, L>(x, lo, inv);
      if constexpr (BITS == 3) {
        x0[k][rho >> 2] += (uint32_t)(p & 3) << (8 * bb + 2 * (rho & 3));
        x1[k][rho >> 3] += (uint32_t)((p >> 2) & 1) << (8 * bb + (rho & 7));
      } else {
        x0[k][rho / P0] += (uint32_t)p << (8 * bb + W0 * (rho % P0));
      }
    }
  }
  if constexpr (BITS != 3) {
    constexpr uint32_t corr = (uint32_t)MAGIC * field_bit_sum(W0);
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
    for (int j = 0; j < 2 * W0; ++j) x0[k][j] = quad_transpose(x0[k][j], sa, sb);
    if constexpr (BITS == 3) {
      x1[k][0] = quad_transpose(x1[k][0], sa, sb);
      x1[k][1] = quad_transpose(x1[k][1], sa, sb);
    }
  }
  if (!valid) return;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int pos = (2 * beta + k + 2 * (quad & 3)) & 7;
    if constexpr (W0 == 2) {
      *reinterpret_cast<uint4*>(quad0 + 16 * pos) = make_uint4(x0[k][0], x0[k][1], x0[k][2], x0[k][3]);
    } else {
      *reinterpret_cast<uint4*>(quad0 + 16 * pos) = make_uint4(x0[k][0], x0[k][1], x0[k][2], x0[k][3]);
      *reinterpret_cast<uint4*>(quad0 + 128 + 16 * pos) =
          make_uint4(x0[k][4], x0[k][5], x0[k][6], x0[k][7]);
    }
    if constexpr (BITS == 3)
      *reinterpret_cast<uint2*>(quad1 + 8 * pos) = make_uint2(x1[k][0], x1[k][1]);
  }
}

struct TileInfo {
  int u;        // unit (sequence, KV head)
  int pk0;      // packed index of the tile's first row
  int nv;       // valid rows (multiple of 4)
  int z;        // input row of the tile's first token: b * n_tok + token - n0
};

__device__ __forceinline__ TileInfo tile_info(const PrefillArgs& a, int h, int l) {
  const int b = l / a.tiles_per_unit, i = l - b * a.tiles_per_unit;
  TileInfo t;
  t.u = b * a.c.n_kv_heads + h;
  t.pk0 = a.pa + TILE * i;
  t.nv = min(TILE, a.pb - t.pk0);
  t.z = b * a.n_tok + (int)((int64_t)a.c.sink + t.pk0 - a.n0);
  return t;
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity,
                                              volatile int* abort_flag) {
  for (uint32_t i = 0; i < PF_WAIT_POLLS; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 63u && *abort_flag) return false;
  }
  return false;
}

__device__ __forceinline__ void raise_abort(volatile int* abort_flag, int* status) {
  *abort_flag = 1;
  atomicOr(status, DEV_ERR_TIMEOUT);
}

template <int BITS, bool AFFINE>
__global__ void __launch_bounds__(NTHREADS, 1)
    prefill_tc_kernel(const __grid_constant__ PrefillArgs a, const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint64_t* k_full = bars + 0;    // [2]
  uint64_t* k_empty = bars + 2;   // [2]
  uint64_t* v_full = bars + 4;    // [2]
  uint64_t* v_empty = bars + 6;   // [2]
  uint64_t* t_full = bars + 8;    // [2] accumulator ready
  uint64_t* t_empty = bars + 10;  // [2] accumulator drained
  uint64_t* drain = bars + 12;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_MISC + 4);

  const DevCache& c = a.c;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x / a.ctas_per_head, share = blockIdx.x % a.ctas_per_head;
  const int n_head_tiles = c.units / c.n_kv_heads * a.tiles_per_unit;
  const int t_begin = (int)((int64_t)n_head_tiles * share / a.ctas_per_head);
  const int t_end = (int)((int64_t)n_head_tiles * (share + 1) / a.ctas_per_head);
  const int nt = t_end - t_begin;
  if (nt <= 0) return;

  // ---- setup: T split into bf16 hi + mid + lo, swizzled K-major ------------
  {
    const float4* T4 = reinterpret_cast<const float4*>(a.T + (size_t)h * D * D);
    for (int q = tid; q < D * D / 4; q += NTHREADS) {
      const int i = q >> 5, j0 = (q & 31) * 4;
      const float4 v = __ldg(T4 + q);
      const float vv[4] = {v.x, v.y, v.z, v.w};
      uint32_t part[3][2];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        // each remainder is exact in fp32 (the difference of a float and
        // its bf16 rounding)
        const __nv_bfloat16 b0 = __float2bfloat16_rn(vv[e]);
        const float r1 = vv[e] - __bfloat162float(b0);
        const __nv_bfloat16 b1 = __float2bfloat16_rn(r1);
        const __nv_bfloat16 b2 = __float2bfloat16_rn(r1 - __bfloat162float(b1));
        const uint32_t sh = 16u * (e & 1);
        if ((e & 1) == 0) part[0][e >> 1] = part[1][e >> 1] = part[2][e >> 1] = 0u;
        part[0][e >> 1] |= (uint32_t)__bfloat16_as_ushort(b0) << sh;
        part[1][e >> 1] |= (uint32_t)__bfloat16_as_ushort(b1) << sh;
        part[2][e >> 1] |= (uint32_t)__bfloat16_as_ushort(b2) << sh;
      }
      const int off = (j0 >> 6) * HALF_BYTES + i * 128 + ((((j0 & 63) >> 3) ^ (i & 7)) << 4) +
                      (j0 & 7) * 2;
      *reinterpret_cast<uint2*>(sm + OFF_THI + off) = make_uint2(part[0][0], part[0][1]);
      *reinterpret_cast<uint2*>(sm + OFF_TMID + off) = make_uint2(part[1][0], part[1][1]);
      *reinterpret_cast<uint2*>(sm + OFF_TLO + off) = make_uint2(part[2][0], part[2][1]);
    }
    fence_proxy_async();   // generic-proxy writes -> visible to the tensor core
  }
  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 4);
      mbar_init(&t_full[s], 1);
      mbar_init(&t_empty[s], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmk);
    tma_prefetch_desc(&tmv);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ---- TMA producer ---------------------------------------------------------
    if (lane == 0) {
      uint32_t k_issued[2] = {0u, 0u}, v_issued[2] = {0u, 0u};
      for (int j = 0; j < nt; ++j) {
        const int s = j & 1;
        const uint32_t use = (uint32_t)(j >> 1);
        const TileInfo t = tile_info(a, h, t_begin + j);
        if (use > 0 && !wait_or_abort(&k_empty[s], (use - 1) & 1, abort_flag)) {
          raise_abort(abort_flag, c.status);
          break;
        }
        unsigned char* kd = sm + OFF_K + s * TILE_BYTES;
        mbar_arrive_expect_tx(&k_full[s], TILE_BYTES);
        tma_load_3d(kd, &tmk, 0, h, t.z, &k_full[s]);
        tma_load_3d(kd + HALF_BYTES, &tmk, 64, h, t.z, &k_full[s]);
        k_issued[s] = use + 1;
        if (use > 0 && !wait_or_abort(&v_empty[s], (use - 1) & 1, abort_flag)) {
          raise_abort(abort_flag, c.status);
          break;
        }
        unsigned char* vd = sm + OFF_V + s * TILE_BYTES;
        mbar_arrive_expect_tx(&v_full[s], TILE_BYTES);
        tma_load_3d(vd, &tmv, 0, h, t.z, &v_full[s]);
        tma_load_3d(vd + HALF_BYTES, &tmv, 64, h, t.z, &v_full[s]);
        v_issued[s] = use + 1;
      }
      // own copies still in flight (only after an abort) must land first
      for (int s = 0; s < 2; ++s) {
        if (k_issued[s]) mbar_wait_bounded(&k_full[s], (k_issued[s] - 1) & 1, PF_WAIT_POLLS);
        if (v_issued[s]) mbar_wait_bounded(&v_full[s], (v_issued[s] - 1) & 1, PF_WAIT_POLLS);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---- MMA issuer -------------------------------------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16(true, TILE, D);
      // smallest terms first
      const uint32_t tpart[3] = {smem_addr(sm + OFF_TLO), smem_addr(sm + OFF_TMID),
                                 smem_addr(sm + OFF_THI)};
      for (int j = 0; j < nt; ++j) {
        const int s = j & 1;
        const uint32_t use = (uint32_t)(j >> 1);
        if (!wait_or_abort(&k_full[s], use & 1, abort_flag)) {
          raise_abort(abort_flag, c.status);
          break;
        }
        if (use > 0 && !wait_or_abort(&t_empty[s], (use - 1) & 1, abort_flag)) {
          raise_abort(abort_flag, c.status);
          break;
        }
        tc_fence_after();
        const uint32_t ka = smem_addr(sm + OFF_K + s * TILE_BYTES);
        const uint32_t dt = tmem_base + (uint32_t)(s * D);
#pragma unroll
        for (int tp = 0; tp < 3; ++tp)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t koff = (uint32_t)((kk >> 2) * HALF_BYTES + (kk & 3) * 32);
            umma_f16_ss(dt, sdesc_kmajor_sw128(ka + koff, 1024),
                        sdesc_kmajor_sw128(tpart[tp] + koff, 1024), idesc,
                        (tp | kk) ? 1u : 0u);
          }
        umma_commit(&k_empty[s]);
        umma_commit(&t_full[s]);
      }
      umma_commit(drain);
      mbar_wait_bounded(drain, 0, PF_WAIT_POLLS);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ---- epilogue warpgroups ------------------------------------------------------
    const int g = (warp - 4) >> 2;
    const int wq = warp & 3;                 // TMEM lane quarter of this warp
    const int row = wq * 32 + lane;          // token row of the tile
    const int beta = row & 3;
    constexpr int W0 = BITS == 3 ? 2 : BITS;
    const bool lo_second = c.r_lo == 2, hi_second = c.r_hi == 127;
    for (int j = g; j < nt; j += 2) {
      const uint32_t use = (uint32_t)(j >> 1);
      const TileInfo t = tile_info(a, h, t_begin + j);
      const bool valid = row < t.nv;
      const int pk = t.pk0 + row;
      const size_t pu0 = (size_t)t.u * c.plane_unit_stride[0];
      const size_t pu1 = (size_t)t.u * c.plane_unit_stride[1];
      uint8_t* kmeta = c.k_meta + (size_t)t.u * c.meta_unit_stride + (size_t)pk * c.meta_bytes;
      uint8_t* vmeta = c.v_meta + (size_t)t.u * c.meta_unit_stride + (size_t)pk * c.meta_bytes;
      __half2 xh[64];
      float lo = 0.f, inv;
      uint32_t meta;

      // K': TMEM lane `row`, 128 fp32 columns -> fp16
      bool ok = wait_or_abort(&t_full[g], use & 1, abort_flag);
      if (!__all_sync(FULL, ok)) {
        raise_abort(abort_flag, c.status);
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + (uint32_t)(g * D) + ((uint32_t)(wq * 32) << 16);
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t r[32];
        tmem_ld32(taddr + (uint32_t)(cc * 32), r);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e)
          xh[cc * 16 + e] = __floats2half2_rn(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&t_empty[g]);
      if (valid) {
        if constexpr (AFFINE) affine_params(xh, BITS, lo_second, hi_second, lo, inv, meta);
        else quest_params(xh, BITS, c.alpha, inv, meta);
        emit_k_row<BITS, AFFINE>(xh, lo, inv, c.k_plane[0] + pu0 + (size_t)pk * 16 * W0,
                                 BITS == 3 ? c.k_plane[1] + pu1 + (size_t)pk * 16 : nullptr);
        if constexpr (AFFINE) *reinterpret_cast<uint32_t*>(kmeta) = meta;
        else *reinterpret_cast<uint16_t*>(kmeta) = (uint16_t)meta;
      }

      // V: swizzled bf16 row from the smem tile -> fp16
      ok = wait_or_abort(&v_full[g], use & 1, abort_flag);
      if (!__all_sync(FULL, ok)) {
        raise_abort(abort_flag, c.status);
        break;
      }
      {
        const unsigned char* vs = sm + OFF_V + g * TILE_BYTES + row * 128;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const uint4 q = *reinterpret_cast<const uint4*>(vs + hf * HALF_BYTES + ((ch ^ (row & 7)) << 4));
            const int e = hf * 32 + ch * 4;
            xh[e] = bf16x2_to_h2(q.x);
            xh[e + 1] = bf16x2_to_h2(q.y);
            xh[e + 2] = bf16x2_to_h2(q.z);
            xh[e + 3] = bf16x2_to_h2(q.w);
          }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&v_empty[g]);
      // every lane of the warp takes part in the quad transposes
      if constexpr (AFFINE) affine_params(xh, BITS, lo_second, hi_second, lo, inv, meta);
      else quest_params(xh, BITS, c.alpha, inv, meta);
      const int quad = pk >> 2;
      emit_v_quad<BITS, AFFINE>(xh, lo, inv, beta, quad,
                                c.v_plane[0] + pu0 + (size_t)quad * 64 * W0,
                                BITS == 3 ? c.v_plane[1] + pu1 + (size_t)quad * 64 : nullptr, valid);
      if (valid) {
        if constexpr (AFFINE) *reinterpret_cast<uint32_t*>(vmeta) = meta;
        else *reinterpret_cast<uint16_t*>(vmeta) = (uint16_t)meta;
      }
    }
  }
  // warps 2 and 3 have no role after the setup

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 256);
  }
}

}  // namespace

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn lookup_encode() {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<EncodeTiledFn>(p);
}

// [rows][Hkv][128] bf16 rows, box = 128 rows x 64 dims of one head,
// 128-byte swizzle (the K-major operand layout of the MMA).
bool make_row_map(CUtensorMap* m, const void* base, int n_kv_heads, int64_t rows) {
  static const EncodeTiledFn encode = lookup_encode();
  if (!encode) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)n_kv_heads, (cuuint64_t)rows};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)n_kv_heads * D * 2};
  const cuuint32_t box[3] = {64, 1, (cuuint32_t)TILE};
  const cuuint32_t estr[3] = {1, 1, 1};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BITS, bool AFFINE>
cudaError_t launch_t(const PrefillArgs& a, const CUtensorMap& mk, const CUtensorMap& mv,
                     unsigned grid, cudaStream_t s) {
  int dev = 0;
  cudaGetDevice(&dev);
  static int attr_done[64] = {0};
  if (dev < 64 && !attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel<BITS, AFFINE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_done[dev] = 1;
  }
  prefill_tc_kernel<BITS, AFFINE><<<grid, NTHREADS, SMEM_BYTES, s>>>(a, mk, mv);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_tc(const PrefillArgs& a, const void* k, const void* v, int sms,
                              cudaStream_t s) {
  const int B = a.c.units / a.c.n_kv_heads;
  CUtensorMap mk, mv;
  if (!make_row_map(&mk, k, a.c.n_kv_heads, (int64_t)B * a.n_tok) ||
      !make_row_map(&mv, v, a.c.n_kv_heads, (int64_t)B * a.n_tok))
    return cudaErrorInvalidValue;
  const unsigned grid = (unsigned)(a.c.n_kv_heads * a.ctas_per_head);
  (void)sms;
  const bool aff = a.c.quantizer == WUSHKV_AFFINE_PCTCLIP;
  switch (a.c.bits) {
    case 2: return aff ? launch_t<2, true>(a, mk, mv, grid, s) : launch_t<2, false>(a, mk, mv, grid, s);
    case 3: return aff ? launch_t<3, true>(a, mk, mv, grid, s) : launch_t<3, false>(a, mk, mv, grid, s);
    case 4: return aff ? launch_t<4, true>(a, mk, mv, grid, s) : launch_t<4, false>(a, mk, mv, grid, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace wushkv
