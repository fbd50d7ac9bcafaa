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
// One CTA (4 warps) per (unit, tile of 64 (query, head) rows: 64 / G queries
// times the G heads of the unit's group).  The CTA walks the unit's tokens in
// blocks of up to 64 of one kind -- sink rows, one packed block record, ring
// rows -- and stages each block in shared memory as fp16 rows: window rows
// as stored, packed tokens as their codes (small integers, exact in fp16),
// with a per-token (scale, offset) pair for keys and for values, so that
//   score_t = scale_t (q . row_t) + offset_t sum(q)
//   out    += (p_t vscale_t) vrow_t + p_t voffset_t
// equal the dequantised products (QuEST: scale = delta, offset = -delta (L/2
// - 1/2) with rows = codes; affine: scale = s, offset = lo).  Scores and PV
// run on fp16 mma.sync m16n8k16 with fp32 accumulation, the query as fp16
// hi + lo terms (about 22 bits); online softmax in base 2 per row, the P
// fragments reused from the score accumulators.
#include <cuda_fp16.h>

#include "async_copy.cuh"
#include "decode_frag.cuh"
#include "wushkv_internal.cuh"

namespace wushkv {

namespace {

constexpr int PA_ROWS = 64;        // (query, head) rows per CTA
constexpr int PA_TOK = 64;         // tokens per staged block
constexpr int PA_LD = D + 8;       // halves per shared row (272 bytes: conflict-free ldmatrix)

struct PaSmem {
  __half qhi[PA_ROWS][PA_LD], qlo[PA_ROWS][PA_LD];
  __half kr[PA_TOK][PA_LD], vr[PA_TOK][PA_LD];
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

// Rows [0, cnt) of a block of fp16 window rows (sink or ring) into kr / vr;
// rows past cnt are zero.  Scales 1, offsets 0.
__device__ __forceinline__ void stage_window(const PaArgs& a, PaSmem& sh, int u, int kind, int t0, int cnt,
                                             int tid) {
  const DevCache& c = a.c;
  for (int e = tid; e < 2 * PA_TOK * 16; e += 128) {
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
    *reinterpret_cast<uint4*>(&(kv ? sh.vr : sh.kr)[i][8 * ch]) = val;
  }
  if (tid < PA_TOK) {
    const bool ok = tid < cnt;
    sh.ks[tid] = ok ? 1.f : 0.f;
    sh.ko[tid] = 0.f;
    sh.vs[tid] = ok ? 1.f : 0.f;
    sh.vo[tid] = 0.f;
  }
}

// Tokens [0, cnt) of packed block record blk into kr / vr as code values
// (plane by plane: the second plane of 3-bit codes adds 4 x its bit), and
// their (scale, offset) pairs; rows past cnt are zero.
__device__ __forceinline__ void stage_packed(const PaArgs& a, PaSmem& sh, int u, int blk, int cnt, int tid) {
  const DevCache& c = a.c;
  const uint64_t boff = block_offset(c, u, blk);
  for (int p = 0; p < c.n_planes; ++p) {
    const int w = c.plane_bits[p], F = 8 / w;
    const uint32_t mask = (1u << w) - 1u;
    const float mul = p == 0 ? 1.f : 4.f;
    const uint8_t* kb = c.k_plane[p] + boff;
    const uint8_t* vb = c.v_plane[p] + boff;
    // K rows: 4w words per token row (row position swizzled within the block)
    for (int e = tid; e < PA_TOK * 4 * w; e += 128) {
      const int i = e / (4 * w), wi = e % (4 * w);
      uint32_t word = 0u;
      if (i < cnt) word = __ldg(reinterpret_cast<const uint32_t*>(kb + (size_t)k_row_pos(i) * 16 * w) + wi);
      for (int beta = 0; beta < 4; ++beta)
        for (int s = 0; s < F; ++s) {
          const float v = (float)((word >> (8 * beta + w * s)) & mask) * mul;
          __half* dst = &sh.kr[i][k_field_dim(wi, w, s, beta)];
          *dst = p == 0 ? __float2half_rn(v) : __float2half_rn(__half2float(*dst) + v);
        }
    }
    // V quads: 16 quads of 4 tokens, 16w words each (row units rotated per quad)
    for (int e = tid; e < 16 * 8 * 2 * w; e += 128) {
      const int q = e / (16 * w), rj = e % (16 * w), r = rj / (2 * w), j = rj % (2 * w);
      uint32_t word = 0u;
      if (4 * q < cnt)
        word = __ldg(reinterpret_cast<const uint32_t*>(vb + (size_t)q * 64 * w) +
                     v_word_index(q, r, j, w));   // the block starts at a multiple of 16 quads
      for (int s = 0; s < F; ++s) {
        const int dim = v_field_dim(r * 2 * w + j, w, s);
        for (int beta = 0; beta < 4; ++beta) {
          const int i = 4 * q + beta;
          const float v = i < cnt ? (float)((word >> (8 * beta + w * s)) & mask) * mul : 0.f;
          __half* dst = &sh.vr[i][dim];
          *dst = p == 0 ? __float2half_rn(v) : __float2half_rn(__half2float(*dst) + v);
        }
      }
    }
    __syncthreads();   // the second plane adds to what the first wrote
  }
  if (tid < PA_TOK) {
    float ks = 0.f, ko = 0.f, vs = 0.f, vo = 0.f;
    if (tid < cnt) {
      const __half* km = reinterpret_cast<const __half*>(c.k_meta + boff + (size_t)tid * c.meta_bytes);
      const __half* vm = reinterpret_cast<const __half*>(c.v_meta + boff + (size_t)tid * c.meta_bytes);
      if (c.quantizer == WUSHKV_AFFINE_PCTCLIP) {
        ks = __half2float(km[0]); ko = __half2float(km[1]);
        vs = __half2float(vm[0]); vo = __half2float(vm[1]);
      } else {
        const float off = (float)(1 << (c.bits - 1)) - 0.5f;   // bin centres (code - L/2 + 1/2) delta
        ks = __half2float(km[0]); ko = -ks * off;
        vs = __half2float(vm[0]); vo = -vs * off;
      }
    }
    sh.ks[tid] = ks; sh.ko[tid] = ko; sh.vs[tid] = vs; sh.vo[tid] = vo;
  }
}

template <int G>
__global__ void __launch_bounds__(128) prefill_attn_kernel(const __grid_constant__ PaArgs a) {
  extern __shared__ __align__(16) unsigned char pa_smem[];
  PaSmem& sh = *reinterpret_cast<PaSmem*>(pa_smem);
  constexpr int QT = PA_ROWS / G;   // queries per tile
  const DevCache& c = a.c;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gq = lane >> 2, c4 = lane & 3;
  const int u = blockIdx.y, b = u / c.n_kv_heads, h = u - b * c.n_kv_heads;
  const int q0 = blockIdx.x * QT;
  const int nq_tile = min(QT, a.n_q - q0);
  const int Hq = c.n_kv_heads * G;

  // q' and the cache may come from the kernel launched just before this one
  grid_dependency_wait();
  grid_dependents_may_launch();

  // ---- query rows R = qi G + g: fp16 hi + lo terms, and sum(q) per row ----------
  for (int e = tid; e < PA_ROWS * 32; e += 128) {   // one row per warp iteration
    const int R = e >> 5, d4 = e & 31, qi = R / G, g = R % G;
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (qi < nq_tile)
      x = __ldg(reinterpret_cast<const float4*>(a.q + (((size_t)b * a.n_q + q0 + qi) * Hq + h * G + g) * D) + d4);
    const float xs[4] = {x.x, x.y, x.z, x.w};
    __half hi[4], lo[4];
    for (int k = 0; k < 4; ++k) {
      hi[k] = __float2half_rn(xs[k]);
      lo[k] = __float2half_rn(xs[k] - __half2float(hi[k]));
    }
    *reinterpret_cast<uint2*>(&sh.qhi[R][4 * d4]) = *reinterpret_cast<const uint2*>(hi);
    *reinterpret_cast<uint2*>(&sh.qlo[R][4 * d4]) = *reinterpret_cast<const uint2*>(lo);
    float sum = (x.x + x.y) + (x.z + x.w);
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) sh.qsum[R] = sum;
  }

  // this thread's two rows (gq and gq + 8 of the warp's 16)
  int pos[2];
  bool rvalid[2];
  for (int k = 0; k < 2; ++k) {
    const int R = 16 * warp + gq + 8 * k, qi = R / G;
    rvalid[k] = qi < nq_tile;
    pos[k] = a.n - a.n_q + q0 + qi;
  }
  const int pmax = a.n - a.n_q + q0 + nq_tile - 1;

  float O[16][4];
  for (int nt = 0; nt < 16; ++nt) O[nt][0] = O[nt][1] = O[nt][2] = O[nt][3] = 0.f;
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f}, ev[2] = {0.f, 0.f};

  const int n_rec = a.n - a.ns - a.P;
  const int nb_sink = (a.ns + PA_TOK - 1) / PA_TOK, nb_pk = (a.P + PA_TOK - 1) / PA_TOK;
  const int nblocks = nb_sink + nb_pk + (n_rec + PA_TOK - 1) / PA_TOK;
  const uint32_t qaddr_hi = smem_addr(&sh.qhi[16 * warp + (lane & 15)][8 * (lane >> 4)]);
  const uint32_t qaddr_lo = smem_addr(&sh.qlo[16 * warp + (lane & 15)][8 * (lane >> 4)]);
  const uint32_t kaddr = smem_addr(&sh.kr[(lane & 7) + 8 * (lane >> 4)][8 * ((lane >> 3) & 1)]);
  const uint32_t vaddr = smem_addr(&sh.vr[(lane & 7) + 8 * ((lane >> 3) & 1)][8 * (lane >> 4)]);

  for (int ib = 0; ib < nblocks; ++ib) {
    int kind, t0, cnt;
    if (ib < nb_sink) {
      kind = 0; t0 = PA_TOK * ib; cnt = min(PA_TOK, a.ns - t0);
    } else if (ib < nb_sink + nb_pk) {
      kind = 1; const int j = ib - nb_sink; t0 = a.ns + PA_TOK * j; cnt = min(PA_TOK, a.P - PA_TOK * j);
    } else {
      kind = 2; const int j = ib - nb_sink - nb_pk; t0 = a.ns + a.P + PA_TOK * j; cnt = min(PA_TOK, n_rec - PA_TOK * j);
    }
    if (t0 > pmax) break;   // every later token is after every query of the tile
    __syncthreads();        // the previous block's rows have been read
    if (kind == 1) stage_packed(a, sh, u, ib - nb_sink, cnt, tid);
    else stage_window(a, sh, u, kind, t0, cnt, tid);
    __syncthreads();

    // ---- scores: 16 rows x 64 tokens per warp -------------------------------------
    float S[8][4];
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
        const int R = 16 * warp + gq + 8 * k;
        const bool ok = rvalid[k] && tl < cnt && t0 + tl <= pos[k];
        const float x = ok ? a.scale_log2 * fmaf(sh.ks[tl], S[nt][e], sh.ko[tl] * sh.qsum[R]) : -INFINITY;
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
        ldmatrix_x4_trans(bv, vaddr + kt * 16 * PA_LD * 2 + dp * 32);
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

template <int G>
cudaError_t launch_g(const PaArgs& a, cudaStream_t s) {
  auto k = prefill_attn_kernel<G>;
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
  return launch_with_overlap(k, grid, dim3(128), (size_t)smem, s, a);
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
