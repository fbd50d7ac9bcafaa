// Bulk (prefill) append of keys on the fifth-generation tensor cores.
//
// Method source: summary page "WUSH-KV：数据自适应变换的 KV Cache 低比特量化"
// (ai-papers-daily), sections 工作参考价值 and 方法关键点: keys are multiplied by
// the per-head transform after RoPE (K' = K T^T for a block of tokens), and
// every token vector that leaves the fp16 recent window is quantised per
// token (QuEST INT or percentile-clipped affine) and bit-packed.  This file
// handles the key rows of one append from its first quad boundary on: each
// goes to the fp16 sink, the packed cache or the fp16 recent ring by its
// token index.  The value rows go through the value-pack kernel; the flush
// of old ring rows and a partial first quad stay with the FMA append kernel.
//
// Design (one CTA per SM, 20 warps, all tiles of a CTA from one KV head):
//   warp 0      TMA producer: 128-token bf16 K tiles (128-byte swizzle)
//               through a four-stage shared-memory ring;
//   warps 4-7   converters, one per TMEM lane quarter: thread i reads token
//               row i of a landed tile, rounds it to fp16 (bf16 values inside
//               the fp16 range are exact; below 2^-17 they round to the fp16
//               grid, an error far under the transform's) and stores it into
//               one of two TMEM operand buffers (64 columns, row i in lane i),
//               freeing the shared-memory stage at once;
//   warp 1      tensor-memory owner and MMA issuer: K' 2^s = K T_lo^T +
//               K T_hi^T with A = K from tensor memory and B = T from shared
//               memory, T 2^s = T_hi + T_lo split into two fp16 matrices (s a
//               per-head power of two putting max |T| 2^s in [2^13, 2^14), so
//               T is kept to about 2^-22 relative, as close to the exact
//               product as an fp32 FMA loop); fp32 accumulation in three
//               128-column TMEM accumulators.  Two fp16 terms take 16 MMAs a
//               tile where three bf16 terms would take 24 (a 128x128x16 MMA
//               runs ~94 cycles here); A in tensor memory keeps the MMAs'
//               shared-memory reads to T alone;
//   warps 8-19  three epilogue warpgroups taking every third tile; thread i
//               owns token row i (TMEM lane i): pass 1 reads its 128 fp32
//               columns in two 64-column loads, rounds K' = acc 2^-s to fp16,
//               takes the
//               per-token statistics and writes the fp16 row back into TMEM;
//               pass 2 reads the fp16 row in double-buffered 16-column blocks
//               for the codes, placed two at a time into the packed words.
// Every wait is bounded; on a timeout the CTA records DEV_ERR_TIMEOUT, stops
// issuing, waits (bounded) for its own copies and MMAs, frees TMEM and ends.
#include <cuda.h>

#include "wushkv_internal.cuh"
#include "tcgen05.cuh"
#include "quant_row.cuh"

namespace wushkv {

namespace {

using namespace rowq;

constexpr int TILE = 128;                    // tokens per tile (MMA M)
constexpr int NSTAGE = 4;                    // bf16 K tiles in shared memory
constexpr int NACC = 3;                      // TMEM accumulators = epilogue warpgroups
constexpr int NABUF = 2;                     // TMEM fp16 operand buffers
constexpr int CONV_WARP = 4;                 // converters: warps 4-7 (lane quarters 0-3)
constexpr int FIRST_EPI_WARP = 8;
constexpr int NTHREADS = (FIRST_EPI_WARP + 4 * NACC) * 32;
constexpr int TMEM_COLS = 512;
constexpr int ABUF_COL = NACC * D;           // operand buffers after the accumulators
constexpr int ABUF_COLS = D / 2;             // 128 fp16 per lane = 64 columns
static_assert(ABUF_COL + NABUF * ABUF_COLS <= TMEM_COLS, "tensor memory columns");
constexpr int TILE_BYTES = TILE * D * 2;     // one bf16 tile, 32 KB
constexpr int HALF_BYTES = TILE_BYTES / 2;   // 64 dims (one 128-byte swizzle span)
constexpr uint32_t PF_WAIT_POLLS = 1u << 22;

// shared memory map (offsets from a 1024-byte aligned base)
constexpr int OFF_THI = 0;
constexpr int OFF_TLO = OFF_THI + TILE_BYTES;
constexpr int OFF_K = OFF_TLO + TILE_BYTES;
constexpr int OFF_BAR = OFF_K + NSTAGE * TILE_BYTES;
constexpr int N_BARS = 2 * NSTAGE + 2 * NABUF + 2 * NACC + 1;
constexpr int OFF_MISC = OFF_BAR + 8 * N_BARS;
constexpr int SMEM_USED = OFF_MISC + 16;   // tmem slot, abort flag, max |T|
constexpr int SMEM_BYTES = SMEM_USED + 1024;          // slack for the alignment
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");

struct TileInfo {
  int u;        // unit (sequence, KV head)
  int t0;       // absolute token of the tile's first row
  int nv;       // valid rows
  int z;        // input row of the tile's first token: b * n_tok + t0 - n0
};

__device__ __forceinline__ TileInfo tile_info(const PrefillArgs& a, int h, int l) {
  const int b = l / a.tiles_per_unit, i = l - b * a.tiles_per_unit;
  TileInfo t;
  t.u = b * a.c.n_kv_heads + h;
  t.t0 = a.ta + TILE * i;
  t.nv = min(TILE, a.tb - t.t0);
  t.z = b * a.n_tok + (int)(t.t0 - a.n0);
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

// Row modes of the epilogue
enum : int { ROW_NONE = 0, ROW_PACKED = 1, ROW_FP16 = 2 };

// fp16 values of two accumulator columns: K' = accumulator * 2^-s (exact),
// rounded once to fp16.
__device__ __forceinline__ uint32_t kprime_h2(uint32_t a, uint32_t b, float2 unscale) {
  const float2 v = mul2_rn(make_float2(__uint_as_float(a), __uint_as_float(b)), unscale);
  const __half2 h = __floats2half2_rn(v.x, v.y);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Codes of column block cc (dims 32 cc .. 32 cc + 31, ks = cc) from its 16
// fp16 pairs into the row's packed words.
template <int BITS, bool AFFINE>
__device__ __forceinline__ void key_block(const uint32_t (&hb)[16], int cc, const QParams& q,
                                          uint32_t (&w0)[8], uint32_t (&w1)[4], uint32_t (&t4)[8],
                                          bool packed, uint8_t* row0) {
  constexpr int L = 1 << BITS;
  const uint32_t m2 = 1u << (2 * cc), m4 = 1u << (4 * (cc & 1)), m1 = 1u << cc;
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const int i = 2 * e;                                 // dim within the block: 16 h + 4 c + beta
    const int hh = i >> 4, cq = (i >> 2) & 3, beta = i & 3;   // beta in {0, 2}
    const __half2 x2 = *reinterpret_cast<const __half2*>(&hb[e]);
    const uint2 p = code_pat2<AFFINE, L>(x2, q);
    // codes to bytes beta, beta + 1; byte 1 of a pattern is zero
    const uint32_t placed = __byte_perm(p.x, p.y, beta == 0 ? 0x1140u : 0x4011u);
    if constexpr (BITS == 2) {
      w0[2 * cq + hh] += placed * m2;
    } else if constexpr (BITS == 3) {
      w0[2 * cq + hh] += (placed & 0x03030303u) * m2;
      w1[cq] += ((placed >> 2) & 0x01010101u) * (m1 << (4 * hh));
    } else {
      t4[2 * cq + hh] += placed * m4;
    }
  }
  if constexpr (BITS == 4) {
    // words 4 c + 2 h + cc / 2 are complete after the odd block
    if (cc & 1) {
      if (packed) {
        uint32_t* o = reinterpret_cast<uint32_t*>(row0);
#pragma unroll
        for (int xw = 0; xw < 8; ++xw) o[2 * xw + (cc >> 1)] = t4[xw];
      }
#pragma unroll
      for (int xw = 0; xw < 8; ++xw) t4[xw] = 0u;
    }
  }
}

// Packed words of the row from its fp16 K' (TMEM columns 0-63, two dims per
// column): four blocks of 16 columns, each load issued while the previous
// block is processed.
template <int BITS, bool AFFINE>
__device__ __forceinline__ void key_codes(uint32_t taddr, const QParams& q, bool packed,
                                          uint32_t (&w0)[8], uint32_t (&w1)[4], uint8_t* row0) {
  uint32_t t4[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) t4[i] = 0u;
  uint32_t ra[16], rb[16];
  tmem_ld16(taddr, ra);
#pragma unroll 1
  for (int cp = 0; cp < 2; ++cp) {
    tmem_wait_ld();                                          // block 2 cp in ra
    tmem_ld16(taddr + (uint32_t)(32 * cp + 16), rb);
    key_block<BITS, AFFINE>(ra, 2 * cp, q, w0, w1, t4, packed, row0);
    tmem_wait_ld();                                          // block 2 cp + 1 in rb
    if (cp == 0) tmem_ld16(taddr + 32u, ra);
    key_block<BITS, AFFINE>(rb, 2 * cp + 1, q, w0, w1, t4, packed, row0);
  }
}

// Key row of one token from its TMEM lane.  Pass 1 reads the fp32
// accumulator in two 64-column loads, rounds K' = acc 2^-s to fp16, takes the
// per-token statistics, stores fp16 windows rows (ROW_FP16) to `win` and
// writes the fp16 row back into the (already read) columns 0-63.  Pass 2
// (warps with a ROW_PACKED lane) turns the fp16 row into codes (packed
// format of wushkv.h): dim d = 32 ks + 4 c + 16 h + beta goes to word
// c w + rho / (8/w), field rho mod (8/w), byte beta, with rho = 4 h + ks; the
// two codes of a pair (beta, beta + 1) share a word and a field and are
// placed together with one byte permute.  At 2 bits the four lanes holding a
// quad's rows then exchange fields so that each stores its share of the
// quad's words (K quads: field = token).  Every lane of the warp must call
// (the TMEM accesses and the exchange are warp-wide).
template <int BITS, bool AFFINE>
__device__ __forceinline__ void key_row(uint32_t taddr, float2 unscale, double alpha,
                                        bool lo_second, bool hi_second, int mode, uint8_t* row0,
                                        uint8_t* row1, uint8_t* meta_p, __half* win, int64_t quad) {
  const bool packed = mode == ROW_PACKED;
  AffineStats ast;
  QuestStats qst;
  ast.init();
  qst.init();
#pragma unroll 1
  for (int hf = 0; hf < 2; ++hf) {
    uint32_t r[64];
    tmem_ld64(taddr + (uint32_t)(64 * hf), r);
    tmem_wait_ld();
    uint32_t hb[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) hb[e] = kprime_h2(r[2 * e], r[2 * e + 1], unscale);
    if constexpr (AFFINE) {
#pragma unroll
      for (int e = 0; e < 16; ++e)
        ast.add2(*reinterpret_cast<const __half2*>(&hb[2 * e]),
                 *reinterpret_cast<const __half2*>(&hb[2 * e + 1]));
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) qst.add(*reinterpret_cast<const __half2*>(&hb[e]));
    }
    if (mode == ROW_FP16) {
      uint4* o = reinterpret_cast<uint4*>(win + 64 * hf);
#pragma unroll
      for (int v = 0; v < 8; ++v) o[v] = make_uint4(hb[4 * v], hb[4 * v + 1], hb[4 * v + 2], hb[4 * v + 3]);
    }
    tmem_st32(taddr + (uint32_t)(32 * hf), hb);
  }
  tmem_wait_st();
  if (!__any_sync(FULL, packed)) return;

  QParams q;
  if constexpr (AFFINE) affine_finish(ast, BITS, lo_second, hi_second, q);
  else quest_finish(qst, BITS, alpha, q);
  uint32_t w0[8], w1[4];
#pragma unroll
  for (int i = 0; i < 8; ++i) w0[i] = 0u;
#pragma unroll
  for (int i = 0; i < 4; ++i) w1[i] = 0u;
  key_codes<BITS, AFFINE>(taddr, q, packed, w0, w1, row0);
  if constexpr (BITS == 2) {
    // 2-bit keys are stored in quads of 4 tokens (the four lanes 4k .. 4k + 3
    // hold a quad's rows): word (c, h) of lane f holds k-step ks at field ks;
    // the quad's word omega = 8 ks + 4 h + c holds token f at field f.  Lane
    // f collects the words of k-step f from the four lanes.
    // A 4 x 4 transpose of 2-bit fields (lane f, field ks) -> (lane ks,
    // field f) in two exchange rounds: with lane f ^ 1 the fields of the
    // other parity, then with lane f ^ 2 the other half of each byte.
    const int f = threadIdx.x & 3;
    uint32_t qw[8];
#pragma unroll
    for (int x = 0; x < 8; ++x) {   // x = 2 c + h
      const uint32_t X = w0[x];
      const uint32_t P = __shfl_xor_sync(FULL, X, 1);
      const uint32_t Xa = (f & 1) ? (((P & 0xCCCCCCCCu) >> 2) | (X & 0xCCCCCCCCu))
                                  : ((X & 0x33333333u) | ((P & 0x33333333u) << 2));
      const uint32_t Q = __shfl_xor_sync(FULL, Xa, 2);
      qw[x] = (f & 2) ? (((Q & 0xF0F0F0F0u) >> 4) | (Xa & 0xF0F0F0F0u))
                      : ((Xa & 0x0F0F0F0Fu) | ((Q & 0x0F0F0F0Fu) << 4));
    }
    if (!packed) return;
    uint32_t* o = reinterpret_cast<uint32_t*>(row0);   // the quad's 128 bytes
#pragma unroll
    for (int x = 0; x < 8; ++x) o[k2_word_pos(quad, 8 * f + 4 * (x & 1) + (x >> 1))] = qw[x];
  }
  if (!packed) return;
  if constexpr (BITS == 3) {
    uint4* o0 = reinterpret_cast<uint4*>(row0);
    o0[0] = make_uint4(w0[0], w0[1], w0[2], w0[3]);
    o0[1] = make_uint4(w0[4], w0[5], w0[6], w0[7]);
  }
  if constexpr (BITS == 3) *reinterpret_cast<uint4*>(row1) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
  if constexpr (AFFINE) *reinterpret_cast<uint32_t*>(meta_p) = q.meta;
  else *reinterpret_cast<uint16_t*>(meta_p) = (uint16_t)q.meta;
}

template <int BITS, bool AFFINE>
__global__ void __launch_bounds__(NTHREADS, 1)
    prefill_tc_kernel(const __grid_constant__ PrefillArgs a, const __grid_constant__ CUtensorMap tmk) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint64_t* k_full = bars;                                // [NSTAGE] bf16 tile landed
  uint64_t* k_empty = bars + NSTAGE;                      // [NSTAGE] tile read by the converters
  uint64_t* a_full = bars + 2 * NSTAGE;                   // [NABUF] fp16 operand in TMEM
  uint64_t* a_empty = bars + 2 * NSTAGE + NABUF;          // [NABUF] operand consumed by the MMAs
  uint64_t* t_full = bars + 2 * NSTAGE + 2 * NABUF;       // [NACC] accumulator ready
  uint64_t* t_empty = t_full + NACC;                      // [NACC] accumulator drained
  uint64_t* drain = t_empty + NACC;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_MISC + 4);
  unsigned int* tmax_bits = reinterpret_cast<unsigned int*>(sm + OFF_MISC + 8);

  const DevCache& c = a.c;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x / a.ctas_per_head, share = blockIdx.x % a.ctas_per_head;
  const int n_head_tiles = c.units / c.n_kv_heads * a.tiles_per_unit;
  const int t_begin = (int)((int64_t)n_head_tiles * share / a.ctas_per_head);
  const int t_end = (int)((int64_t)n_head_tiles * (share + 1) / a.ctas_per_head);
  const int nt = t_end - t_begin;
  if (nt <= 0) return;

  // ---- setup: T 2^s = T_hi + T_lo in fp16, swizzled K-major ----------------
  const float4* T4 = reinterpret_cast<const float4*>(a.T + (size_t)h * D * D);
  if (tid == 0) *tmax_bits = 0u;
  __syncthreads();
  {
    float m = 0.f;
    for (int qd = tid; qd < D * D / 4; qd += NTHREADS) {
      const float4 v = __ldg(T4 + qd);
      m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
    m = warp_max_f32(m);
    if (lane == 0) atomicMax(tmax_bits, __float_as_uint(m));   // non-negative: bits order as values
  }
  __syncthreads();
  // 2^s with max |T| 2^s in [2^13, 2^14)
  int s_exp = 0;
  {
    const float tmax = __uint_as_float(*tmax_bits);
    if (tmax > 0.f && isfinite(tmax)) {
      int e;
      frexpf(tmax, &e);                      // tmax = f 2^e, f in [0.5, 1)
      s_exp = min(max(14 - e, -100), 100);   // a near-zero T keeps a finite scale
    }
  }
  const float scale = ldexpf(1.f, s_exp);
  const float2 unscale = make_float2(ldexpf(1.f, -s_exp), ldexpf(1.f, -s_exp));
  for (int qd = tid; qd < D * D / 4; qd += NTHREADS) {
    const int i = qd >> 5, j0 = (qd & 31) * 4;
    const float4 v = __ldg(T4 + qd);
    const float vv[4] = {v.x * scale, v.y * scale, v.z * scale, v.w * scale};   // exact
    uint32_t part[2][2];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      // the remainder is exact in fp32 (a float minus its fp16 rounding)
      const __half b0 = __float2half_rn(vv[e]);
      const __half b1 = __float2half_rn(vv[e] - __half2float(b0));
      const uint32_t sh = 16u * (e & 1);
      if ((e & 1) == 0) part[0][e >> 1] = part[1][e >> 1] = 0u;
      part[0][e >> 1] |= (uint32_t)__half_as_ushort(b0) << sh;
      part[1][e >> 1] |= (uint32_t)__half_as_ushort(b1) << sh;
    }
    const int off = (j0 >> 6) * HALF_BYTES + i * 128 + ((((j0 & 63) >> 3) ^ (i & 7)) << 4) +
                    (j0 & 7) * 2;
    *reinterpret_cast<uint2*>(sm + OFF_THI + off) = make_uint2(part[0][0], part[0][1]);
    *reinterpret_cast<uint2*>(sm + OFF_TLO + off) = make_uint2(part[1][0], part[1][1]);
  }
  fence_proxy_async();   // generic-proxy writes -> visible to the tensor core
  if (tid == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 4);
    }
    for (int b = 0; b < NABUF; ++b) {
      mbar_init(&a_full[b], 4);
      mbar_init(&a_empty[b], 1);
    }
    for (int g = 0; g < NACC; ++g) {
      mbar_init(&t_full[g], 1);
      mbar_init(&t_empty[g], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmk);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ---- TMA producer ---------------------------------------------------------
    if (lane == 0) {
      uint32_t issued[NSTAGE] = {0u, 0u, 0u, 0u};
      for (int j = 0; j < nt; ++j) {
        const int s = j % NSTAGE;
        const uint32_t use = (uint32_t)(j / NSTAGE);
        const TileInfo t = tile_info(a, h, t_begin + j);
        if (use > 0 && !wait_or_abort(&k_empty[s], (use - 1) & 1, abort_flag)) {
          raise_abort(abort_flag, c.status);
          break;
        }
        unsigned char* kd = sm + OFF_K + s * TILE_BYTES;
        mbar_arrive_expect_tx(&k_full[s], TILE_BYTES);
        tma_load_3d(kd, &tmk, 0, h, t.z, &k_full[s]);
        tma_load_3d(kd + HALF_BYTES, &tmk, 64, h, t.z, &k_full[s]);
        issued[s] = use + 1;
      }
      // own copies still in flight (only after an abort) must land first
      for (int s = 0; s < NSTAGE; ++s)
        if (issued[s]) mbar_wait_bounded(&k_full[s], (issued[s] - 1) & 1, PF_WAIT_POLLS);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---- MMA issuer -------------------------------------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16(false, TILE, D);   // fp16 x fp16 -> fp32
      const uint32_t tpart[2] = {smem_addr(sm + OFF_TLO), smem_addr(sm + OFF_THI)};  // small first
      for (int j = 0; j < nt; ++j) {
        const int ab = j % NABUF, acc = j % NACC;
        const uint32_t use_a = (uint32_t)(j / NABUF), use_t = (uint32_t)(j / NACC);
        if (!wait_or_abort(&a_full[ab], use_a & 1, abort_flag)) {
          raise_abort(abort_flag, c.status);
          break;
        }
        if (use_t > 0 && !wait_or_abort(&t_empty[acc], (use_t - 1) & 1, abort_flag)) {
          raise_abort(abort_flag, c.status);
          break;
        }
        tc_fence_after();
        const uint32_t at = tmem_base + (uint32_t)(ABUF_COL + ab * ABUF_COLS);
        const uint32_t dt = tmem_base + (uint32_t)(acc * D);
#pragma unroll
        for (int tp = 0; tp < 2; ++tp)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t koff = (uint32_t)((kk >> 2) * HALF_BYTES + (kk & 3) * 32);
            umma_f16_ts(dt, at + (uint32_t)(8 * kk), sdesc_kmajor_sw128(tpart[tp] + koff, 1024),
                        idesc, (tp | kk) ? 1u : 0u);
          }
        umma_commit(&a_empty[ab]);
        umma_commit(&t_full[acc]);
      }
      umma_commit(drain);
      mbar_wait_bounded(drain, 0, PF_WAIT_POLLS);
    }
    __syncwarp();
  } else if (warp < CONV_WARP) {
    // warps 2 and 3 have no role after the setup
  } else if (warp < FIRST_EPI_WARP) {
    // ---- converters: bf16 row -> fp16 row in a TMEM operand buffer ------------
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    for (int j = 0; j < nt; ++j) {
      const int s = j % NSTAGE, ab = j % NABUF;
      const uint32_t use_s = (uint32_t)(j / NSTAGE), use_a = (uint32_t)(j / NABUF);
      bool ok = wait_or_abort(&k_full[s], use_s & 1, abort_flag);
      if (ok && use_a > 0) ok = wait_or_abort(&a_empty[ab], (use_a - 1) & 1, abort_flag);
      if (!__all_sync(FULL, ok)) {
        raise_abort(abort_flag, c.status);
        break;
      }
      tc_fence_after();
      uint32_t r[64];
      const unsigned char* src = sm + OFF_K + s * TILE_BYTES + row * 128;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf)
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint4 q4 = *reinterpret_cast<const uint4*>(src + hf * HALF_BYTES + ((ch ^ (row & 7)) << 4));
          const __half2 h0 = bf16x2_to_h2(q4.x), h1 = bf16x2_to_h2(q4.y);
          const __half2 h2 = bf16x2_to_h2(q4.z), h3 = bf16x2_to_h2(q4.w);
          const int e = hf * 32 + ch * 4;
          r[e] = *reinterpret_cast<const uint32_t*>(&h0);
          r[e + 1] = *reinterpret_cast<const uint32_t*>(&h1);
          r[e + 2] = *reinterpret_cast<const uint32_t*>(&h2);
          r[e + 3] = *reinterpret_cast<const uint32_t*>(&h3);
        }
      tmem_st64(tmem_base + (uint32_t)(ABUF_COL + ab * ABUF_COLS) + lane_off, r);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&a_full[ab]);
        mbar_arrive(&k_empty[s]);
      }
    }
  } else {
    // ---- epilogue warpgroups ------------------------------------------------------
    const int g = (warp - FIRST_EPI_WARP) >> 2;   // accumulator of this group
    const int wq = warp & 3;                 // TMEM lane quarter of this warp
    const int row = wq * 32 + lane;          // token row of the tile
    const bool lo_second = c.r_lo == 2, hi_second = c.r_hi == 127;
    const uint32_t taddr = tmem_base + (uint32_t)(g * D) + ((uint32_t)(wq * 32) << 16);
    for (int j = g; j < nt; j += NACC) {
      const uint32_t use = (uint32_t)(j / NACC);
      const TileInfo t = tile_info(a, h, t_begin + j);
      // destination of this row by its token index
      const int tok = t.t0 + row;
      const int pk = tok - c.sink;
      int mode = ROW_NONE;
      __half* win = nullptr;
      if (row < t.nv) {
        if (tok < c.sink) {
          mode = ROW_FP16;
          win = c.sink_k + ((size_t)t.u * c.sink + tok) * D;
        } else if (pk < a.packed1) {
          mode = ROW_PACKED;
        } else {
          mode = ROW_FP16;
          win = c.ring_k + ((size_t)t.u * c.ring_slots + (size_t)(pk % c.ring_slots)) * D;
        }
      }
      const size_t pkc = mode == ROW_PACKED ? (size_t)pk : 0;
      const bool ok = wait_or_abort(&t_full[g], use & 1, abort_flag);
      if (!__all_sync(FULL, ok)) {
        raise_abort(abort_flag, c.status);
        break;
      }
      tc_fence_after();
      // (packed destinations are looked up only for packed rows)
      const bool pkd = mode == ROW_PACKED;
      key_row<BITS, AFFINE>(
          taddr, unscale, c.alpha, lo_second, hi_second, mode,
          pkd ? (BITS == 2 ? k_quad_at(c, t.u, (int64_t)pkc / 4) : k_row_at(c, 0, t.u, (int64_t)pkc)) : nullptr,
          (BITS == 3 && pkd) ? k_row_at(c, 1, t.u, (int64_t)pkc) : nullptr,
          pkd ? k_meta_at(c, t.u, (int64_t)pkc) : nullptr, win, (int64_t)pkc / 4);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&t_empty[g]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
namespace {

// [rows][Hkv][128] bf16 rows, box = 128 rows x 64 dims of one head,
// 128-byte swizzle (the K-major operand layout of the MMA).
bool make_row_map(CUtensorMap* m, const void* base, int n_kv_heads, int64_t rows) {
  const EncodeTiledFn encode = tensor_map_encoder();
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
cudaError_t launch_t(const PrefillArgs& a, const CUtensorMap& mk, unsigned grid, cudaStream_t s) {
  int dev = 0;
  cudaGetDevice(&dev);
  static int attr_done[64] = {0};
  if (dev < 64 && !attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel<BITS, AFFINE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_done[dev] = 1;
  }
  prefill_tc_kernel<BITS, AFFINE><<<grid, NTHREADS, SMEM_BYTES, s>>>(a, mk);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_tc(const PrefillArgs& a, const void* k, const void* v, int sms,
                              cudaStream_t s) {
  const int B = a.c.units / a.c.n_kv_heads;
  CUtensorMap mk;
  if (!make_row_map(&mk, k, a.c.n_kv_heads, (int64_t)B * a.n_tok)) return cudaErrorInvalidValue;
  const unsigned grid = (unsigned)(a.c.n_kv_heads * a.ctas_per_head);
  const bool aff = a.c.quantizer == WUSHKV_AFFINE_PCTCLIP;
  cudaError_t e;
  switch (a.c.bits) {
    case 2: e = aff ? launch_t<2, true>(a, mk, grid, s) : launch_t<2, false>(a, mk, grid, s); break;
    case 3: e = aff ? launch_t<3, true>(a, mk, grid, s) : launch_t<3, false>(a, mk, grid, s); break;
    case 4: e = aff ? launch_t<4, true>(a, mk, grid, s) : launch_t<4, false>(a, mk, grid, s); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  return launch_value_pack(a, v, sms, s);
}

}  // namespace wushkv
