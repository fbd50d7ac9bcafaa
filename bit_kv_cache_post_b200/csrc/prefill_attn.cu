// Chunked-prefill attention over the quantised cache.
//
// The pages describe decoding only; prefill attention is the cache's second
// consumer, built with the decode's reading (summary page "WUSH-KV：数据自适应
// 变换的 KV Cache 低比特量化", 方法关键点: keys transformed after RoPE, queries
// through T^-T; a query attends after its own token was appended): the chunk's
// n_q tokens are the last n_q tokens of every sequence and have been appended
// first, and the query of token p = n - n_q + i attends to tokens 0 .. p as
// the cache holds them (fp16 sink and recent rows, dequantised packed
// tokens).
//
// One CTA (8 warps) per (unit, tile of 128 (query, head) rows: 128 / G
// queries times the G heads of the unit's group).  The CTA walks the unit's tokens in
// blocks of up to 64 of one kind -- sink rows, one packed block record, ring
// rows -- and stages each block in shared memory as fp16 rows: window rows
// as stored, packed tokens as their codes (small integers, exact in fp16),
// with a per-token (scale, offset) pair for keys and for values, so that
//   score_t = scale_t (q . row_t) + offset_t sum(q)
//   out    += (p_t vscale_t) vrow_t + p_t voffset_t
// equal the dequantised products (key rows = codes, value rows = codes -
// (L - 1) / 2; QuEST: scale = delta, key offset = -delta (L - 1) / 2, value
// offset 0; affine: scale = s, key offset = lo, value offset = lo + s (L -
// 1) / 2).  Scores and PV
// run on fp16 mma.sync m16n8k16 with fp32 accumulation, the query as fp16
// hi + lo terms (about 22 bits); online softmax in base 2 per row, the P
// fragments reused from the score accumulators.  The raw words of the next
// packed block record load into registers while the current block is used.
#include <cuda_fp16.h>

#include "async_copy.cuh"
#include "decode_frag.cuh"
#include "wushkv_internal.cuh"

namespace wushkv {

namespace {

constexpr int PA_WARPS = 8;
constexpr int PA_THREADS = PA_WARPS * 32;
constexpr int PA_ROWS = 16 * PA_WARPS;   // (query, head) rows per CTA
constexpr int PA_TOK = 64;               // tokens per staged block (one packed block record)
constexpr int PA_LD = D + 8;             // halves per shared row (272 bytes: conflict-free ldmatrix)
constexpr int PA_LDT = PA_TOK + 8;       // halves per transposed value row (144 bytes)

struct PaSmem {
  __half qhi[PA_ROWS][PA_LD], qlo[PA_ROWS][PA_LD];
  __half kr[PA_TOK][PA_LD];      // key rows [token][dim]
  __half vt[D][PA_LDT];          // value rows transposed [dim][token]
  float ks[PA_TOK], ko[PA_TOK], vs[PA_TOK], vo[PA_TOK];
  float qsum[PA_ROWS];
};

__device__ __forceinline__ float pa_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Plane widths of a code width: 2 -> {2}, 3 -> {2, 1}, 4 -> {4}.
template <int BITS> struct Planes {
  static constexpr int N = BITS == 3 ? 2 : 1;
  static constexpr int W0 = BITS == 4 ? 4 : 2;
  static constexpr int W1 = BITS == 3 ? 1 : 0;
  // words a thread holds for one block record: per plane 64 x 4w K words and
  // 16 x 16w V words over PA_THREADS threads
  static constexpr int K0 = PA_TOK * 4 * W0 / PA_THREADS, V0 = 16 * 16 * W0 / PA_THREADS;
  static constexpr int K1 = PA_TOK * 4 * W1 / PA_THREADS, V1 = 16 * 16 * W1 / PA_THREADS;
};

// The raw words of one packed block record that this thread decodes: K row
// words (token e / 4w, word e % 4w) and V quad words (quad e / 16w, row unit,
// unit word), e = tid + PA_THREADS j; plus the meta of token tid.
template <int BITS>
struct RawBlock {
  using PL = Planes<BITS>;
  uint32_t k0[PL::K0], v0[PL::V0];
  uint32_t k1[PL::K1 > 0 ? PL::K1 : 1], v1[PL::V1 > 0 ? PL::V1 : 1];
  uint32_t km, vm;
};

template <int BITS>
__device__ __forceinline__ void load_block(const DevCache& c, int u, int blk, int cnt, int tid, RawBlock<BITS>& r) {
  using PL = Planes<BITS>;
  const uint64_t boff = block_offset(c, u, blk);
#pragma unroll
  for (int p = 0; p < PL::N; ++p) {
    const int w = p == 0 ? PL::W0 : PL::W1;
    const uint8_t* kb = c.k_plane[p] + boff;
    const uint8_t* vb = c.v_plane[p] + boff;
#pragma unroll
    for (int j = 0; j < (p == 0 ? PL::K0 : PL::K1); ++j) {
      const int e = tid + PA_THREADS * j;
      uint32_t x;
      if constexpr (BITS == 2) {   // K quads: quad e / 32, word omega = e % 32
        const int q = e >> 5, om = e & 31;
        x = 4 * q < cnt ? __ldg(reinterpret_cast<const uint32_t*>(kb + (size_t)q * 128) + k2_word_pos(q, om)) : 0u;
      } else {
        const int i = e / (4 * w), wi = e % (4 * w);
        x = i < cnt ? __ldg(reinterpret_cast<const uint32_t*>(kb + (size_t)k_row_pos(i) * 16 * w) + wi) : 0u;
      }
      if (p == 0) r.k0[j] = x; else r.k1[j] = x;
    }
#pragma unroll
    for (int j = 0; j < (p == 0 ? PL::V0 : PL::V1); ++j) {
      const int e = tid + PA_THREADS * j, q = e / (16 * w), rj = e % (16 * w);
      const uint32_t x = 4 * q < cnt ? __ldg(reinterpret_cast<const uint32_t*>(vb + (size_t)q * 64 * w) +
                                             v_word_index(q, rj / (2 * w), rj % (2 * w), w))
                                     : 0u;   // the block starts at a multiple of 16 quads
      if (p == 0) r.v0[j] = x; else r.v1[j] = x;
    }
  }
  r.km = r.vm = 0u;
  if (tid < cnt) {
    if (c.meta_bytes == 4) {
      r.km = __ldg(reinterpret_cast<const uint32_t*>(c.k_meta + boff + (size_t)tid * 4));
      r.vm = __ldg(reinterpret_cast<const uint32_t*>(c.v_meta + boff + (size_t)tid * 4));
    } else {
      r.km = __ldg(reinterpret_cast<const unsigned short*>(c.k_meta + boff + (size_t)tid * 2));
      r.vm = __ldg(reinterpret_cast<const unsigned short*>(c.v_meta + boff + (size_t)tid * 2));
    }
  }
}

// The block's codes into kr / vt as fp16 values -- key codes as they are,
// value codes minus (L - 1) / 2 -- (the second plane of 3-bit codes adds
// 4 x its bit after a barrier) and the (scale, offset) pairs; key rows past
// cnt come out zero (their words were loaded as zero), value rows past cnt
// hold -(L - 1) / 2 and get zero weight.
template <int BITS>
__device__ __forceinline__ void write_block(const DevCache& c, PaSmem& sh, int cnt, int tid, const RawBlock<BITS>& r) {
  using PL = Planes<BITS>;
  constexpr float CMID = 0.5f * (float)((1 << BITS) - 1);   // (L - 1) / 2
#pragma unroll
  for (int p = 0; p < PL::N; ++p) {
    const int w = p == 0 ? PL::W0 : PL::W1, F = 8 / w;
    const uint32_t mask = (1u << w) - 1u;
    const float mul = p == 0 ? 1.f : 4.f;
#pragma unroll
    for (int j = 0; j < (p == 0 ? PL::K0 : PL::K1); ++j) {
      const int e = tid + PA_THREADS * j;
      const uint32_t word = p == 0 ? r.k0[j] : r.k1[j];
      if constexpr (BITS == 2) {   // K quads: field f = token 4q + f, byte beta = dim 4 omega + beta
        const int q = e >> 5, om = e & 31;
#pragma unroll
        for (int f = 0; f < 4; ++f) {   // dims 4 omega .. 4 omega + 3 of token 4q + f: one 8-byte store
          const __half2 lo = __floats2half2_rn((float)((word >> (2 * f)) & 3u), (float)((word >> (8 + 2 * f)) & 3u));
          const __half2 hi = __floats2half2_rn((float)((word >> (16 + 2 * f)) & 3u), (float)((word >> (24 + 2 * f)) & 3u));
          uint2 pk;
          pk.x = *reinterpret_cast<const uint32_t*>(&lo);
          pk.y = *reinterpret_cast<const uint32_t*>(&hi);
          *reinterpret_cast<uint2*>(&sh.kr[4 * q + f][4 * om]) = pk;
        }
      } else {
        const int i = e / (4 * w), wi = e % (4 * w);
#pragma unroll
        for (int beta = 0; beta < 4; ++beta)
#pragma unroll
          for (int s = 0; s < F; ++s) {
            const float v = (float)((word >> (8 * beta + w * s)) & mask) * mul;
            __half* dst = &sh.kr[i][k_field_dim(wi, w, s, beta)];
            *dst = p == 0 ? __float2half_rn(v) : __float2half_rn(__half2float(*dst) + v);
          }
      }
    }
#pragma unroll
    for (int j = 0; j < (p == 0 ? PL::V0 : PL::V1); ++j) {
      const int e = tid + PA_THREADS * j, q = e / (16 * w), rj = e % (16 * w);
      const uint32_t word = p == 0 ? r.v0[j] : r.v1[j];
#pragma unroll
      for (int s = 0; s < F; ++s) {
        const int dim = v_field_dim(rj, w, s);
        // the quad's four tokens of this dim (bytes 0..3): one 8-byte store;
        // value codes centred on the grid's middle (the first plane takes the
        // shift): half the magnitude, so P's fp16 rounding counts half
        float v[4];
#pragma unroll
        for (int beta = 0; beta < 4; ++beta)
          v[beta] = (float)((word >> (8 * beta + w * s)) & mask) * mul - (p == 0 ? CMID : 0.f);
        uint2* dst = reinterpret_cast<uint2*>(&sh.vt[dim][4 * q]);
        if (p != 0) {   // the second plane adds to the first
          const uint2 old = *dst;
          const float2 o01 = __half22float2(*reinterpret_cast<const __half2*>(&old.x));
          const float2 o23 = __half22float2(*reinterpret_cast<const __half2*>(&old.y));
          v[0] += o01.x; v[1] += o01.y; v[2] += o23.x; v[3] += o23.y;
        }
        const __half2 lo = __floats2half2_rn(v[0], v[1]), hi = __floats2half2_rn(v[2], v[3]);
        uint2 pk;
        pk.x = *reinterpret_cast<const uint32_t*>(&lo);
        pk.y = *reinterpret_cast<const uint32_t*>(&hi);
        *dst = pk;
      }
    }
    if (PL::N > 1 && p == 0) __syncthreads();   // the second plane adds to what the first wrote
  }
  if (tid < PA_TOK) {
    float ks = 0.f, ko = 0.f, vs = 0.f, vo = 0.f;
    if (tid < cnt) {
      const __half2 kh = *reinterpret_cast<const __half2*>(&r.km);
      const __half2 vh = *reinterpret_cast<const __half2*>(&r.vm);
      ks = __low2float(kh);
      vs = __low2float(vh);
      if (c.quantizer == WUSHKV_AFFINE_PCTCLIP) {   // lo + s code = (lo + s CMID) + s (code - CMID)
        ko = __high2float(kh);
        vo = fmaf(vs, CMID, __high2float(vh));
      } else {   // bin centres (code - L/2 + 1/2) delta = delta (code - CMID)
        ko = -ks * CMID;
        vo = 0.f;
      }
    }
    sh.ks[tid] = ks; sh.ko[tid] = ko; sh.vs[tid] = vs; sh.vo[tid] = vo;
  }
}

// Rows [0, cnt) of a block of fp16 window rows (sink or ring) into kr / vt;
// rows past cnt are zero.  Scales 1, offsets 0.
__device__ __forceinline__ void stage_window(const DevCache& c, PaSmem& sh, int u, int kind, int t0, int cnt,
                                             int tid) {
  for (int e = tid; e < 2 * PA_TOK * 16; e += PA_THREADS) {
    const int kv = e / (PA_TOK * 16), i = (e / 16) % PA_TOK, ch = e % 16;
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (i < cnt) {
      const int t = t0 + i;
      const __half* row;
      if (kind == 0) {
        row = (kv ? c.sink_v : c.sink_k) + ((size_t)u * c.sink + t) * D;
      } else {
        const int slot = (t - c.sink) % c.ring_slots;
        row = (kv ? c.ring_v : c.ring_k) + ((size_t)u * c.ring_slots + slot) * D;
      }
      val = __ldg(reinterpret_cast<const uint4*>(row) + ch);
    }
    if (kv == 0) {
      *reinterpret_cast<uint4*>(&sh.kr[i][8 * ch]) = val;
    } else {   // values transposed: dims 8 ch .. 8 ch + 7 of token i
      const __half* hv = reinterpret_cast<const __half*>(&val);
#pragma unroll
      for (int k = 0; k < 8; ++k) sh.vt[8 * ch + k][i] = hv[k];
    }
  }
  if (tid < PA_TOK) {
    const bool ok = tid < cnt;
    sh.ks[tid] = ok ? 1.f : 0.f;
    sh.ko[tid] = 0.f;
    sh.vs[tid] = ok ? 1.f : 0.f;
    sh.vo[tid] = 0.f;
  }
}

// Kind, first token and token count of block ib of the unit: sink rows,
// then one block per packed record, then ring rows.
struct BlockSpan { int kind, t0, cnt, blk; };
__device__ __forceinline__ BlockSpan block_span(const PaArgs& a, int ib, int nb_sink, int nb_pk, int n_rec) {
  BlockSpan sp;
  sp.blk = 0;
  if (ib < nb_sink) {
    sp.kind = 0; sp.t0 = PA_TOK * ib; sp.cnt = min(PA_TOK, a.ns - sp.t0);
  } else if (ib < nb_sink + nb_pk) {
    sp.kind = 1; sp.blk = ib - nb_sink; sp.t0 = a.ns + PA_TOK * sp.blk; sp.cnt = min(PA_TOK, a.P - PA_TOK * sp.blk);
  } else {
    const int j = ib - nb_sink - nb_pk;
    sp.kind = 2; sp.t0 = a.ns + a.P + PA_TOK * j; sp.cnt = min(PA_TOK, n_rec - PA_TOK * j);
  }
  return sp;
}

template <int G, int BITS>
__global__ void __launch_bounds__(PA_THREADS) prefill_attn_kernel(const __grid_constant__ PaArgs a) {
  extern __shared__ __align__(16) unsigned char pa_smem[];
  PaSmem& sh = *reinterpret_cast<PaSmem*>(pa_smem);
  constexpr int QT = PA_ROWS / G;   // queries per tile
  const DevCache& c = a.c;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gq = lane >> 2, c4 = lane & 3;
  const int u = blockIdx.y, b = u / c.n_kv_heads, h = u - b * c.n_kv_heads;
  const int q0 = blockIdx.x * QT;
  const int nq_tile = min(QT, a.n_q - q0);
  const int Hq = c.n_kv_heads * G;
  const int pmax = a.n - a.n_q + q0 + nq_tile - 1;
  const int n_rec = a.n - a.ns - a.P;
  const int nb_sink = (a.ns + PA_TOK - 1) / PA_TOK, nb_pk = (a.P + PA_TOK - 1) / PA_TOK;
  const int nblocks = nb_sink + nb_pk + (n_rec + PA_TOK - 1) / PA_TOK;

  // q' and the cache may come from the kernel launched just before this one
  grid_dependency_wait();
  grid_dependents_may_launch();

  // the first packed block's words go out before the query rows are prepared
  RawBlock<BITS> raw;
  int raw_ib = -1;
  for (int ib = 0; ib < nblocks; ++ib) {
    const BlockSpan sp = block_span(a, ib, nb_sink, nb_pk, n_rec);
    if (sp.t0 > pmax) break;
    if (sp.kind == 1) { load_block<BITS>(c, u, sp.blk, sp.cnt, tid, raw); raw_ib = ib; break; }
  }

  // ---- query rows R = qi G + g: fp16 hi + lo terms, and sum(q) per row ----------
  for (int e = tid; e < PA_ROWS * 32; e += PA_THREADS) {   // one row per warp iteration
    const int R = e >> 5, d4 = e & 31, qi = R / G, g = R % G;
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (qi < nq_tile)
      x = __ldg(reinterpret_cast<const float4*>(a.q + (((size_t)b * a.n_q + q0 + qi) * Hq + h * G + g) * D) + d4);
    const float xs[4] = {x.x, x.y, x.z, x.w};
    __half hi[4], lo[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      hi[k] = __float2half_rn(xs[k]);
      lo[k] = __float2half_rn(xs[k] - __half2float(hi[k]));
    }
    *reinterpret_cast<uint2*>(&sh.qhi[R][4 * d4]) = *reinterpret_cast<const uint2*>(hi);
    *reinterpret_cast<uint2*>(&sh.qlo[R][4 * d4]) = *reinterpret_cast<const uint2*>(lo);
    float sum = (x.x + x.y) + (x.z + x.w);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) sh.qsum[R] = sum;
  }

  // this thread's two rows (gq and gq + 8 of the warp's 16)
  int pos[2];
  bool rvalid[2];
  float qs[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int R = 16 * warp + gq + 8 * k, qi = R / G;
    rvalid[k] = qi < nq_tile;
    pos[k] = a.n - a.n_q + q0 + qi;
  }

  float O[16][4];
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) O[nt][0] = O[nt][1] = O[nt][2] = O[nt][3] = 0.f;
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f}, ev[2] = {0.f, 0.f};

  const uint32_t qaddr_hi = smem_addr(&sh.qhi[16 * warp + (lane & 15)][8 * (lane >> 4)]);
  const uint32_t qaddr_lo = smem_addr(&sh.qlo[16 * warp + (lane & 15)][8 * (lane >> 4)]);
  const uint32_t kaddr = smem_addr(&sh.kr[(lane & 7) + 8 * (lane >> 4)][8 * ((lane >> 3) & 1)]);
  const uint32_t vaddr = smem_addr(&sh.vt[(lane & 7) + 8 * (lane >> 4)][8 * ((lane >> 3) & 1)]);

  for (int ib = 0; ib < nblocks; ++ib) {
    const BlockSpan sp = block_span(a, ib, nb_sink, nb_pk, n_rec);
    if (sp.t0 > pmax) break;   // every later token is after every query of the tile
    __syncthreads();           // the previous block's rows have been read (and the query rows written)
    if (sp.kind == 1) {
      if (raw_ib != ib) load_block<BITS>(c, u, sp.blk, sp.cnt, tid, raw);
      write_block<BITS>(c, sh, sp.cnt, tid, raw);
      raw_ib = -1;
      if (ib + 1 < nb_sink + nb_pk) {   // the next packed block's words load while this one is used
        const BlockSpan nx = block_span(a, ib + 1, nb_sink, nb_pk, n_rec);
        if (nx.t0 <= pmax) { load_block<BITS>(c, u, nx.blk, nx.cnt, tid, raw); raw_ib = ib + 1; }
      }
    } else {
      stage_window(c, sh, u, sp.kind, sp.t0, sp.cnt, tid);
    }
    __syncthreads();
    if (ib == 0) {
#pragma unroll
      for (int k = 0; k < 2; ++k) qs[k] = sh.qsum[16 * warp + gq + 8 * k];
    }

    // ---- scores: 16 rows x 64 tokens per warp -------------------------------------
    float S[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) S[nt][0] = S[nt][1] = S[nt][2] = S[nt][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      uint32_t ah[4], al[4];
      ldmatrix_x4(ah, qaddr_hi + kk * 32);
      ldmatrix_x4(al, qaddr_lo + kk * 32);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t bk[4];
        ldmatrix_x4(bk, kaddr + np * 16 * PA_LD * 2 + kk * 32);
        mma_f16_k16(S[2 * np], ah[0], ah[1], ah[2], ah[3], bk[0], bk[1]);
        mma_f16_k16(S[2 * np], al[0], al[1], al[2], al[3], bk[0], bk[1]);
        mma_f16_k16(S[2 * np + 1], ah[0], ah[1], ah[2], ah[3], bk[2], bk[3]);
        mma_f16_k16(S[2 * np + 1], al[0], al[1], al[2], al[3], bk[2], bk[3]);
      }
    }

    // ---- masked scores in log2 units, online softmax --------------------------------
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int k = e >> 1, tl = 8 * nt + 2 * c4 + (e & 1);
        const bool ok = rvalid[k] && tl < sp.cnt && sp.t0 + tl <= pos[k];
        const float x = ok ? a.scale_log2 * fmaf(sh.ks[tl], S[nt][e], sh.ko[tl] * qs[k]) : -INFINITY;
        S[nt][e] = x;
        mx[k] = fmaxf(mx[k], x);
      }
    float corr[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      mx[k] = fmaxf(mx[k], __shfl_xor_sync(0xffffffffu, mx[k], 1));
      mx[k] = fmaxf(mx[k], __shfl_xor_sync(0xffffffffu, mx[k], 2));
      const float mn = fmaxf(m[k], mx[k]);
      corr[k] = mn == -INFINITY ? 1.f : pa_ex2(m[k] - mn);   // m = -inf: nothing to rescale
      m[k] = mn;
      l[k] *= corr[k];
      ev[k] *= corr[k];
    }
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      O[nt][0] *= corr[0]; O[nt][1] *= corr[0];
      O[nt][2] *= corr[1]; O[nt][3] *= corr[1];
    }
    uint32_t pf[8][2];   // P' = p vscale as fp16 pairs: [n-tile][row half]
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      float pv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int k = e >> 1, tl = 8 * nt + 2 * c4 + (e & 1);
        const float p = m[k] == -INFINITY ? 0.f : pa_ex2(S[nt][e] - m[k]);
        l[k] += p;
        ev[k] = fmaf(p, sh.vo[tl], ev[k]);
        pv[e] = p * sh.vs[tl];
      }
      pf[nt][0] = pack_half2(pv[0], pv[1]);
      pf[nt][1] = pack_half2(pv[2], pv[3]);
    }

    // ---- PV: 16 rows x 128 dims over the 64 tokens --------------------------------
#pragma unroll
    for (int kt = 0; kt < 4; ++kt) {
      const uint32_t a0 = pf[2 * kt][0], a1 = pf[2 * kt][1], a2 = pf[2 * kt + 1][0], a3 = pf[2 * kt + 1][1];
#pragma unroll
      for (int dp = 0; dp < 8; ++dp) {
        uint32_t bv[4];
        ldmatrix_x4(bv, vaddr + dp * 16 * PA_LDT * 2 + kt * 32);
        mma_f16_k16(O[2 * dp], a0, a1, a2, a3, bv[0], bv[1]);
        mma_f16_k16(O[2 * dp + 1], a0, a1, a2, a3, bv[2], bv[3]);
      }
    }
  }

  // ---- normalise and store ---------------------------------------------------------
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    l[k] += __shfl_xor_sync(0xffffffffu, l[k], 1);
    l[k] += __shfl_xor_sync(0xffffffffu, l[k], 2);
    ev[k] += __shfl_xor_sync(0xffffffffu, ev[k], 1);
    ev[k] += __shfl_xor_sync(0xffffffffu, ev[k], 2);
  }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    if (!rvalid[k]) continue;
    const int R = 16 * warp + gq + 8 * k, qi = R / G, g = R % G;
    const float il = 1.f / l[k], eo = ev[k] * il;
    float* dst = a.out + (((size_t)b * a.n_q + q0 + qi) * Hq + h * G + g) * D;
#pragma unroll
    for (int nt = 0; nt < 16; ++nt)
      *reinterpret_cast<float2*>(dst + 8 * nt + 2 * c4) =
          make_float2(fmaf(O[nt][2 * k], il, eo), fmaf(O[nt][2 * k + 1], il, eo));
  }
}

template <int G, int BITS>
cudaError_t launch_gb(const PaArgs& a, cudaStream_t s) {
  auto k = prefill_attn_kernel<G, BITS>;
  const int smem = (int)sizeof(PaSmem);
  int dev = 0;
  cudaGetDevice(&dev);
  static int attr_done[64] = {};
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr_done[dev] = 1;
  }
  constexpr int QT = PA_ROWS / G;
  const dim3 grid((unsigned)((a.n_q + QT - 1) / QT), (unsigned)a.c.units);
  return launch_with_overlap(k, grid, dim3(PA_THREADS), (size_t)smem, s, a);
}

template <int G>
cudaError_t launch_g(const PaArgs& a, cudaStream_t s) {
  switch (a.c.bits) {
    case 2: return launch_gb<G, 2>(a, s);
    case 3: return launch_gb<G, 3>(a, s);
    case 4: return launch_gb<G, 4>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_prefill_attention(const PaArgs& a, cudaStream_t s) {
  switch (a.c.group) {
    case 1: return launch_g<1>(a, s);
    case 2: return launch_g<2>(a, s);
    case 4: return launch_g<4>(a, s);
    case 8: return launch_g<8>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace wushkv
