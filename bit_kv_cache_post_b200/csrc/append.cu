// Append path: key transform after RoPE, fp16 sink/recent windows, chunked
// flush of the recent window into the packed cache with per-token
// quantisation and bit packing.
//
// Method source: summary page "WUSH-KV：数据自适应变换的 KV Cache 低比特量化"
// (ai-papers-daily), sections 工作参考价值 and 方法关键点: the key transform
// follows RMSNorm and RoPE and costs one d x d product per new token; the
// first 64 and the latest 256 tokens stay in fp16; the recent window is
// quantised in chunks of 8 (or 16).
//
// One CTA (128 threads, one per dim) handles a run of 4-token quads of one
// unit (sequence, KV head).  Quads are the packing granule of the V layout,
// so a quad that reaches the packed cache is quantised and packed whole.
#include "wushkv_internal.cuh"

namespace wushkv {

namespace {

constexpr int TT_LD = 129;  // padded row of the transposed transform in smem

__device__ __forceinline__ float load_in(const void* p, int dtype, size_t i) {
  if (dtype == WUSHKV_F16) return __half2float(static_cast<const __half*>(p)[i]);
  if (dtype == WUSHKV_BF16) return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
  return static_cast<const float*>(p)[i];
}

__device__ __forceinline__ float round_f16(float x) { return __half2float(__float2half_rn(x)); }

// Token classes inside one append.
enum : int { TOK_SKIP = 0, TOK_NEW = 1, TOK_FLUSH_OLD = 2 };

// Shared memory of one append CTA: staging vectors first, then (only when
// the CTA stages the transform) T^T.
constexpr size_t APPEND_VEC_BYTES = (size_t)3 * 4 * D * sizeof(float) + 4 * D + 16;

// One append CTA: quads blockIdx-slice bx of unit u.
__device__ __forceinline__ void append_body(const AppendArgs& a, int64_t bx, int u, unsigned char* smem_raw) {
  float* kin = reinterpret_cast<float*>(smem_raw);         // [4][128] raw keys
  float* k16 = kin + 4 * D;                                // [4][128] fp16 keys
  float* v16 = k16 + 4 * D;                                // [4][128] fp16 values
  uint8_t* codes = reinterpret_cast<uint8_t*>(v16 + 4 * D);  // [4][128]
  int* kind_s = reinterpret_cast<int*>(codes + 4 * D);     // [4]
  float* Tt = reinterpret_cast<float*>(smem_raw + APPEND_VEC_BYTES);  // [128][TT_LD] = T^T

  const DevCache& c = a.c;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = u / c.n_kv_heads, h = u % c.n_kv_heads;
  const int64_t n0 = a.n0, n1 = a.n0 + a.n_tok;
  const int64_t S = c.sink, P0 = a.packed0, P1 = a.packed1;
  const int W = c.ring_slots;

  const int64_t q_first = a.quad_begin + bx * a.quads_per_cta;
  const int64_t q_last = min(q_first + a.quads_per_cta, a.quad_begin + a.n_quads);
  if (q_first >= q_last) return;

  // Stage T^T of this head once per CTA if several quads need the product;
  // a single quad reads T's rows directly instead.
  const bool has_new = (4 * q_last > n0) && (4 * q_first < n1);
  const bool transform = (a.T != nullptr) && has_new;
  const bool staged = transform && (q_last - q_first > 1);
  if (staged) stage_transpose_128(a.T + (size_t)h * D * D, Tt, TT_LD);

  for (int64_t Q = q_first; Q < q_last; ++Q) {
    __syncthreads();  // previous quad's smem consumers are done
    // ---- gather the quad's four tokens (all loads in flight at once) --------
    {
      int kind[4];
      float kx[4], vx[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t t = 4 * Q + j;
        kind[j] = TOK_SKIP;
        if (t >= n0 && t < n1) kind[j] = TOK_NEW;
        else if (t < n0 && t >= S + P0 && t < S + P1) kind[j] = TOK_FLUSH_OLD;
        kx[j] = vx[j] = 0.f;
        if (kind[j] == TOK_NEW) {
          const size_t row = (((size_t)b * a.n_tok + (size_t)(t - n0)) * c.n_kv_heads + h) * D;
          kx[j] = load_in(a.k, a.dtype, row + tid);
          vx[j] = load_in(a.v, a.dtype, row + tid);
        } else if (kind[j] == TOK_FLUSH_OLD) {
          const int slot = (int)((t - S) % W);
          const size_t off = ((size_t)u * W + slot) * D + tid;
          kx[j] = __half2float(c.ring_k[off]);
          vx[j] = __half2float(c.ring_v[off]);
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (tid == 0) kind_s[j] = kind[j];
        if (kind[j] == TOK_NEW) {
          kin[j * D + tid] = kx[j];
          v16[j * D + tid] = round_f16(vx[j]);
        } else if (kind[j] == TOK_FLUSH_OLD) {
          k16[j * D + tid] = kx[j];
          v16[j * D + tid] = vx[j];
        }
      }
    }
    __syncthreads();
    // ---- key transform k' = T k (fp32 FMA), one output dim per thread ------
    if (transform && !staged) {
      // rows 32 warp .. 32 warp + 31 in four groups of eight (the same
      // arithmetic as every other single-token and query transform)
      float4 x4[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) x4[j] = *reinterpret_cast<const float4*>(kin + j * D + 4 * lane);
      const int rsel = ((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1);
#pragma unroll 1
      for (int rg = 0; rg < 4; ++rg) {
        float dots[4];
        const int row0 = 32 * warp + 8 * rg;
        matvec_rows8<4>(a.T + (size_t)h * D * D, row0, x4, dots);
        if ((lane & 3) == 0)
          for (int j = 0; j < 4; ++j)
            if (kind_s[j] == TOK_NEW) k16[j * D + row0 + rsel] = round_f16(dots[j]);
      }
    } else {
      for (int j = 0; j < 4; ++j) {
        if (kind_s[j] != TOK_NEW) continue;
        float acc;
        if (transform) {
          acc = 0.f;
          const float* kj = kin + j * D;
#pragma unroll 8
          for (int jj = 0; jj < D; ++jj) acc = fmaf(Tt[jj * TT_LD + tid], kj[jj], acc);
        } else {
          acc = kin[j * D + tid];
        }
        k16[j * D + tid] = round_f16(acc);
      }
    }
    __syncthreads();
    // ---- destinations --------------------------------------------------------
    const int64_t t0 = 4 * Q;
    const bool packed_quad = (t0 >= S) && (t0 + 4 <= S + P1) &&
                             (kind_s[0] | kind_s[1] | kind_s[2] | kind_s[3]) != TOK_SKIP;
    if (!packed_quad) {
      for (int j = 0; j < 4; ++j) {
        if (kind_s[j] != TOK_NEW) continue;
        const int64_t t = t0 + j;
        if (t < S) {
          const size_t off = ((size_t)u * S + (size_t)t) * D + tid;
          c.sink_k[off] = __float2half_rn(k16[j * D + tid]);
          c.sink_v[off] = __float2half_rn(v16[j * D + tid]);
        } else {
          const int slot = (int)((t - S) % W);
          const size_t off = ((size_t)u * W + slot) * D + tid;
          c.ring_k[off] = __float2half_rn(k16[j * D + tid]);
          c.ring_v[off] = __float2half_rn(v16[j * D + tid]);
        }
      }
      continue;
    }
    // ---- quantise + pack a whole quad -------------------------------------------
    const int64_t pk = t0 - S;  // packed index of the quad's first token
    if (pk + 4 > c.packed_capacity) {   // the host's bookkeeping went wrong: never write past the region
      if (tid == 0) atomicOr(c.status, DEV_ERR_RANGE);
      continue;
    }
    for (int kv = 0; kv < 2; ++kv) {
      const float* src = (kv == 0 ? k16 : v16) + warp * D;
      float x[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) x[i] = src[4 * lane + i];
      uint8_t cd[4];
      uint8_t* meta = kv == 0 ? k_meta_at(c, u, pk + warp) : v_meta_at(c, u, pk + warp);
      if (c.quantizer == WUSHKV_QUEST_INT) {
        __half dl;
        quest_warp(x, c.bits, c.alpha, cd, dl);
        if (lane == 0) *reinterpret_cast<__half*>(meta) = dl;
      } else {
        __half s, lo;
        affine_warp(x, c.bits, c.r_lo, c.r_hi, cd, s, lo);
        if (lane == 0) *reinterpret_cast<__half2*>(meta) = __halves2half2(s, lo);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) codes[warp * D + 4 * lane + i] = cd[i];
      __syncthreads();
      for (int p = 0; p < c.n_planes; ++p) {
        const int w = c.plane_bits[p], P = 8 / w;
        if (kv == 0 && c.bits == 2) {
          // one K quad, 32 words: thread tid builds word omega = tid from the
          // four tokens' codes of dims 4 tid .. 4 tid + 3
          if (tid < 32) {
            uint32_t word = 0;
            for (int f = 0; f < 4; ++f)
              for (int beta = 0; beta < 4; ++beta)
                word |= (uint32_t)codes[f * D + 4 * tid + beta] << (8 * beta + 2 * f);
            const int64_t quad = pk / 4;
            reinterpret_cast<uint32_t*>(k_quad_at(c, u, quad))[k2_word_pos(quad, tid)] = word;
          }
        } else if (kv == 0) {
          // four K rows, 4w words each: warp = token, lane = word
          if (lane < 4 * w) {
            uint32_t word = 0;
            for (int s = 0; s < P; ++s)
              for (int beta = 0; beta < 4; ++beta) {
                const int dim = k_field_dim(lane, w, s, beta);
                word |= plane_value(codes[warp * D + dim], c.bits, p) << (8 * beta + w * s);
              }
            reinterpret_cast<uint32_t*>(k_row_at(c, p, u, pk + warp))[lane] = word;
          }
        } else {
          // one V quad, 16w words: thread tid builds unit word (r, j)
          if (tid < 16 * w) {
            const int r = tid / (2 * w), j = tid % (2 * w);
            uint32_t word = 0;
            for (int s = 0; s < P; ++s) {
              const int dim = v_field_dim(tid, w, s);
              for (int beta = 0; beta < 4; ++beta)
                word |= plane_value(codes[beta * D + dim], c.bits, p) << (8 * beta + w * s);
            }
            const int quad = (int)(pk / 4);
            reinterpret_cast<uint32_t*>(v_quad_at(c, p, u, quad))[v_word_index(quad, r, j, w)] = word;
          }
        }
      }
      __syncthreads();
    }
  }
}

__global__ void __launch_bounds__(128, 4) append_kernel(AppendArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  append_body(a, blockIdx.x, blockIdx.y, smem_raw);
}

// The append of a decode step and the query transform of the same step in
// one launch: slices x < gx of row u are the append CTAs of unit u, slice gx
// transforms the unit's G queries.
template <int G>
__global__ void __launch_bounds__(128, G >= 8 ? 3 : 4) append_qt_kernel(AppendArgs a, int gx, const void* q, int q_dtype,
                                                        const float* TinvT, float* q_out) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  // every input and the cache may come from the kernel launched just before;
  // the next kernel is released only after that wait (see grid_dependency_wait)
  grid_dependency_wait();
  grid_dependents_may_launch();
  if ((int)blockIdx.x < gx) {
    append_body(a, blockIdx.x, blockIdx.y, smem_raw);
  } else {
    const int u = blockIdx.y;
    query_transform_unit<G>(q, q_dtype, TinvT, q_out, u / a.c.n_kv_heads, u % a.c.n_kv_heads,
                            a.c.n_kv_heads);
  }
}

// A decode step whose single new token stays in the fp16 windows: row
// slices x < 4 of unit u transform the new key (rows 32x .. 32x + 31 of
// k' = T k) and store those dims of k' and v in the sink or the ring;
// slices 4 .. 7 transform the unit's G queries (rows 32(x - 4) ..); slices
// x >= 8 are the append CTAs of the chunk this step flushes (quads from
// a.quad_begin, no transform).  Each CTA reads only 16 KB of a matrix.
template <int G>
__global__ void __launch_bounds__(128) step_rows_kernel(AppendArgs a, const void* q, int q_dtype,
                                                        const float* TinvT, float* q_out) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  grid_dependency_wait();   // every input and the cache may come from the kernel launched just before
  grid_dependents_may_launch();
  const int x = blockIdx.x, u = blockIdx.y;
  const DevCache& c = a.c;
  const int b = u / c.n_kv_heads, h = u % c.n_kv_heads;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rsel = ((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1);
  if (x >= 8) {
    append_body(a, x - 8, u, smem_raw);
    return;
  }
  const int row0 = 32 * (x & 3) + 8 * warp;
  if (x < 4) {
    const size_t src = ((size_t)b * c.n_kv_heads + h) * D;   // n_tok = 1: [B][1][Hkv][128]
    const int64_t t = a.n0;
    __half* kdst;
    __half* vdst;
    if (t < c.sink) {
      kdst = c.sink_k + ((size_t)u * c.sink + (size_t)t) * D;
      vdst = c.sink_v + ((size_t)u * c.sink + (size_t)t) * D;
    } else {
      const size_t slot = (size_t)((t - c.sink) % c.ring_slots);
      kdst = c.ring_k + ((size_t)u * c.ring_slots + slot) * D;
      vdst = c.ring_v + ((size_t)u * c.ring_slots + slot) * D;
    }
    float y[1];
    if (a.T != nullptr) {
      float4 x4[1] = {load4_any(a.k, a.dtype, src + 4 * lane)};
      matvec_rows8<1>(a.T + (size_t)h * D * D, row0, x4, y);
    } else {
      y[0] = load_in(a.k, a.dtype, src + row0 + rsel);
    }
    if ((lane & 3) == 0) kdst[row0 + rsel] = __float2half_rn(y[0]);
    if (lane < 8) vdst[row0 + lane] = __float2half_rn(load_in(a.v, a.dtype, src + row0 + lane));
  } else {
    const int Hq = c.n_kv_heads * G;
    float4 x4[G];
#pragma unroll
    for (int g = 0; g < G; ++g)
      x4[g] = load4_any(q, q_dtype, ((size_t)b * Hq + (size_t)h * G + g) * D + 4 * lane);
    float y[G];
    matvec_rows8<G>(TinvT + (size_t)h * D * D, row0, x4, y);
    if ((lane & 3) == 0) {
#pragma unroll
      for (int g = 0; g < G; ++g) q_out[((size_t)b * Hq + (size_t)h * G + g) * D + row0 + rsel] = y[g];
    }
  }
}

// Dynamic shared memory of an append launch: T^T only when a CTA transforms
// several quads.
size_t append_smem(const AppendArgs& a) {
  const bool staged = a.T != nullptr && a.quads_per_cta > 1;
  return APPEND_VEC_BYTES + (staged ? (size_t)D * TT_LD * sizeof(float) : 0);
}

cudaError_t set_smem_attr(const void* fn, size_t bytes) {
  return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

}  // namespace

cudaError_t launch_step_rows(const AppendArgs& a, int n_flush_quads, const void* q, int q_dtype,
                             const float* TinvT, float* q_out, cudaStream_t s) {
  const int G = a.c.group;
  dim3 grid((unsigned)(8 + n_flush_quads), (unsigned)a.c.units);
  const size_t smem = APPEND_VEC_BYTES;
  switch (G) {
    case 1: return launch_with_overlap(step_rows_kernel<1>, grid, dim3(128), smem, s, a, q, q_dtype, TinvT, q_out);
    case 2: return launch_with_overlap(step_rows_kernel<2>, grid, dim3(128), smem, s, a, q, q_dtype, TinvT, q_out);
    case 4: return launch_with_overlap(step_rows_kernel<4>, grid, dim3(128), smem, s, a, q, q_dtype, TinvT, q_out);
    case 8: return launch_with_overlap(step_rows_kernel<8>, grid, dim3(128), smem, s, a, q, q_dtype, TinvT, q_out);
    default: return cudaErrorInvalidValue;
  }
}

size_t append_smem_bytes() { return APPEND_VEC_BYTES + (size_t)D * TT_LD * sizeof(float); }

cudaError_t launch_append(const AppendArgs& a, cudaStream_t s) {
  int dev = 0;
  cudaGetDevice(&dev);
  static int attr_done[64] = {0};
  if (dev < 64 && !attr_done[dev]) {
    cudaError_t e = set_smem_attr((const void*)append_kernel, append_smem_bytes());
    if (e != cudaSuccess) return e;
    attr_done[dev] = 1;
  }
  if (a.n_quads <= 0) return cudaSuccess;
  const int64_t gx = (a.n_quads + a.quads_per_cta - 1) / a.quads_per_cta;
  dim3 grid((unsigned)gx, (unsigned)a.c.units);
  append_kernel<<<grid, 128, append_smem(a), s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_append_qt(const AppendArgs& a, const void* q, int q_dtype, const float* TinvT,
                             float* q_out, cudaStream_t s) {
  const int G = a.c.group;
  const void* fn = G == 1 ? (const void*)append_qt_kernel<1> : G == 2 ? (const void*)append_qt_kernel<2>
                   : G == 4 ? (const void*)append_qt_kernel<4> : (const void*)append_qt_kernel<8>;
  int dev = 0;
  cudaGetDevice(&dev);
  static int attr_done[64][4] = {};
  const int gi = G == 1 ? 0 : G == 2 ? 1 : G == 4 ? 2 : 3;
  if (dev < 64 && !attr_done[dev][gi]) {
    cudaError_t e = set_smem_attr(fn, append_smem_bytes());
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    attr_done[dev][gi] = 1;
  }
  const int64_t gx = a.n_quads > 0 ? (a.n_quads + a.quads_per_cta - 1) / a.quads_per_cta : 0;
  dim3 grid((unsigned)gx + 1, (unsigned)a.c.units);
  const size_t smem = append_smem(a);
  switch (G) {
    case 1: return launch_with_overlap(append_qt_kernel<1>, grid, dim3(128), smem, s, a, (int)gx, q, q_dtype, TinvT, q_out);
    case 2: return launch_with_overlap(append_qt_kernel<2>, grid, dim3(128), smem, s, a, (int)gx, q, q_dtype, TinvT, q_out);
    case 4: return launch_with_overlap(append_qt_kernel<4>, grid, dim3(128), smem, s, a, (int)gx, q, q_dtype, TinvT, q_out);
    case 8: return launch_with_overlap(append_qt_kernel<8>, grid, dim3(128), smem, s, a, (int)gx, q, q_dtype, TinvT, q_out);
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace wushkv
