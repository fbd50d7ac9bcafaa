// Internal declarations shared by the libwushkv kernels and host code.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "wushkv.h"

namespace wushkv {

constexpr int D = 128;           // head_dim
constexpr int PARTIAL_FLOATS = D + 4;   // o[128], m, l, 2 pad: one split partial of one head
constexpr unsigned FULL = 0xffffffffu;

// Device-visible view of one cache buffer.  The packed region is a run of
// block records (64 packed tokens each: K planes, V planes, K meta, V meta);
// k_plane[p] etc. point at those parts of unit 0's block 0.
struct DevCache {
  uint8_t* k_plane[2];
  uint8_t* v_plane[2];
  uint64_t unit_stride;              // bytes per unit of the packed region
  uint64_t block_stride;             // bytes per block record
  int n_planes;
  int plane_bits[2];
  int bits;
  int quantizer;
  uint8_t* k_meta;
  uint8_t* v_meta;
  int meta_bytes;                    // 2 (QuEST delta) or 4 (affine scale, lo)
  __half* sink_k;
  __half* sink_v;
  __half* ring_k;
  __half* ring_v;
  int sink, recent, chunk, ring_slots;
  int packed_capacity;
  float* partials;                   // split-K workspace
  int* counters;                     // one arrival counter per unit, counter_stride ints apart
  int counter_stride;
  int max_splits;
  int* status;                       // sticky device error word
  int units, n_kv_heads, group;
  // Paged packed region (null page_table: dense, unit u's blocks at
  // u * unit_stride).  Block blk of sequence b lives in page
  // page_table[b * pt_stride + blk]; a page holds the n_kv_heads block
  // records of that block, head h's at h * block_stride.  Page num_pages is
  // a spare page that out-of-range ids are sent to (and reported).
  const int32_t* page_table;
  int pt_stride, num_pages;
  double alpha;                      // QuEST clip ratio
  int r_lo, r_hi;                    // affine ranks (1-indexed)
};

// Packed tokens per block record.
constexpr int PACK_BLOCK_TOKENS = 64;

// Row position of packed token pk inside its 64-token block: token 8r + j of
// the block sits at row 8r + (j ^ (r & 3)), so that the decode's reads of
// one row per octet r fall on all shared-memory banks.
__host__ __device__ __forceinline__ int k_row_pos(int64_t pk) {
  const int i = (int)(pk & 63);
  return (i & ~7) | ((i & 7) ^ ((i >> 3) & 3));
}

// Byte offset of block record blk of unit u from the start of the packed
// region (the page table's entry when the region is paged).
__device__ __forceinline__ uint64_t block_offset(const DevCache& c, int64_t u, int64_t blk) {
  if (c.page_table == nullptr) return (uint64_t)u * c.unit_stride + (uint64_t)blk * c.block_stride;
  const int64_t b = u / c.n_kv_heads, h = u - b * c.n_kv_heads;
  int page = __ldg(c.page_table + b * c.pt_stride + blk);
  if (page < 0 || page >= c.num_pages) {   // never touch another sequence's page
    atomicOr(c.status, WUSHKV_DEV_RANGE);
    page = c.num_pages;
  }
  return ((uint64_t)page * c.n_kv_heads + (uint64_t)h) * c.block_stride;
}

// 2-bit keys are packed in quads of 4 consecutive tokens (128 bytes, 32
// words): word omega holds dims 4 omega .. 4 omega + 3 at its bytes and token
// 4 quad + f at field f of each byte; with omega = 8 ks + 4 h + c it sits at
// this position of the quad (the decode's lane c reads its eight words of a
// quad as two 16-byte chunks, adjacent quads on alternating chunks).
__host__ __device__ __forceinline__ int k2_word_pos(int64_t quad, int omega) {
  const int ks = omega >> 3, h = (omega >> 2) & 1, c = omega & 3;
  return 4 * ((2 * c + (ks >> 1)) ^ (int)(quad & 1)) + 2 * (ks & 1) + h;
}
// Address of 2-bit K quad `quad` (packed tokens 4 quad .. 4 quad + 3) of unit u.
__device__ __forceinline__ uint8_t* k_quad_at(const DevCache& c, int64_t u, int64_t quad) {
  return c.k_plane[0] + block_offset(c, u, quad >> 4) + (uint64_t)(quad & 15) * 128;
}

// Address of the K row (16 w bytes, plane p) of packed token pk of unit u
// (3- and 4-bit keys).
__device__ __forceinline__ uint8_t* k_row_at(const DevCache& c, int p, int64_t u, int64_t pk) {
  return c.k_plane[p] + block_offset(c, u, pk >> 6) + (uint64_t)k_row_pos(pk) * 16 * c.plane_bits[p];
}
// Address of V quad `quad` (tokens 4 quad .. 4 quad + 3; 64 w bytes, plane p) of unit u.
__device__ __forceinline__ uint8_t* v_quad_at(const DevCache& c, int p, int64_t u, int64_t quad) {
  return c.v_plane[p] + block_offset(c, u, quad >> 4) + (uint64_t)(quad & 15) * 64 * c.plane_bits[p];
}
// Addresses of the per-token meta of packed token pk of unit u.
__device__ __forceinline__ uint8_t* k_meta_at(const DevCache& c, int64_t u, int64_t pk) {
  return c.k_meta + block_offset(c, u, pk >> 6) + (uint64_t)(pk & 63) * c.meta_bytes;
}
__device__ __forceinline__ uint8_t* v_meta_at(const DevCache& c, int64_t u, int64_t pk) {
  return c.v_meta + block_offset(c, u, pk >> 6) + (uint64_t)(pk & 63) * c.meta_bytes;
}

// Window split of one sequence holding n tokens (the cache's policy: sink
// S, recent R, flush chunk C, ring of W = R + C slots), with the decode's
// items: 8-token window chunks and 64-token packed blocks.  Host and device
// use this one definition.
struct SeqGeom {
  int n_sink, n_packed, n_recent, ring_first, win_chunks, pack_blocks;
};
__host__ __device__ __forceinline__ SeqGeom seq_geom(int64_t n, int S, int R, int C, int W) {
  SeqGeom g;
  g.n_sink = (int)(n < S ? n : S);
  const int64_t m = n - g.n_sink;
  g.n_packed = (int)((m >= (int64_t)R + C) ? (int64_t)C * ((m - R) / C) : 0);
  g.n_recent = (int)(m - g.n_packed);
  g.ring_first = W > 0 ? g.n_packed % W : 0;
  g.win_chunks = (g.n_sink + g.n_recent + 7) / 8;
  g.pack_blocks = (g.n_packed + 63) / 64;
  return g;
}

// Status bits a kernel may set in the sticky word (values documented in
// wushkv.h): a packed index past the capacity (the write is skipped), a
// split partial index past the workspace (skipped), a copy that did not
// complete within the wait limit.
enum : int { DEV_ERR_RANGE = WUSHKV_DEV_RANGE, DEV_ERR_SPLITS = WUSHKV_DEV_SPLITS,
             DEV_ERR_TIMEOUT = WUSHKV_DEV_TIMEOUT };

// ---------------------------------------------------------------------------
// Programmatic dependent launch.  A kernel launched with
// launch_with_overlap() may begin while the previous kernel on the stream
// is still running; it must call grid_dependency_wait() before touching
// memory that kernel writes or reads (a no-op when there is no such
// kernel).  grid_dependents_may_launch() lets the next such kernel be
// scheduled; it never skips the wait on the other side.
//
// Every kernel of this library calls grid_dependents_may_launch() only
// after its own grid_dependency_wait(), so at most one kernel before it (its
// immediate predecessor) can still be running when one of them starts.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
}
__device__ __forceinline__ void grid_dependents_may_launch() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_with_overlap(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// ---------------------------------------------------------------------------
// Exact-rounding helpers
// ---------------------------------------------------------------------------

// float64 -> fp16, round to nearest even, rounded once.  Written from the
// IEEE 754 binary16 definition: pick the fp16 quantum (2^(e-10), or 2^-24 in
// the subnormal range), round |x| / quantum to the nearest even integer in
// float64 (exact: power-of-two scaling), and rebuild.  The rebuilt value is
// an fp16 value, so the final float -> half conversion is exact.
__device__ __forceinline__ __half f64_to_f16_rn(double x) {
  double a = fabs(x);
  if (!(a > 0.0)) return __float2half_rn((float)x);          // 0, -0, NaN
  if (a >= 65520.0) return __float2half_rn(x > 0 ? INFINITY : -INFINITY);
  int e = ilogb(a);                                          // floor(log2 a)
  if (e < -14) e = -14;
  double q = rint(ldexp(a, 10 - e));                         // ties to even
  double v = ldexp(q, e - 10);
  return __float2half_rn((float)(x < 0 ? -v : v));
}

__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
  return v;
}

__device__ __forceinline__ float warp_max_f32(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(FULL, v, o));
  return v;
}

// Stage the transpose of a row-major 128 x 128 fp32 matrix into shared
// memory (row stride ld, padded against bank conflicts) with a 128-thread
// block: 16-byte loads, eight in flight per thread.
__device__ __forceinline__ void stage_transpose_128(const float* __restrict__ M, float* Mt, int ld) {
  const float4* M4 = reinterpret_cast<const float4*>(M);
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    float4 v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = __ldg(M4 + threadIdx.x + 128 * (8 * b + k));
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int e = 4 * (threadIdx.x + 128 * (8 * b + k));   // element index
      const int i = e >> 7, j = e & 127;
      Mt[(j + 0) * ld + i] = v[k].x;
      Mt[(j + 1) * ld + i] = v[k].y;
      Mt[(j + 2) * ld + i] = v[k].z;
      Mt[(j + 3) * ld + i] = v[k].w;
    }
  }
}

// Element i of a device array of the given input dtype, as fp32.
__device__ __forceinline__ float load_any(const void* p, int dtype, size_t i) {
  if (dtype == WUSHKV_F16) return __half2float(static_cast<const __half*>(p)[i]);
  if (dtype == WUSHKV_BF16) return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
  return static_cast<const float*>(p)[i];
}

__device__ __forceinline__ float4 load4_any(const void* p, int dtype, size_t i) {
  return make_float4(load_any(p, dtype, i), load_any(p, dtype, i + 1), load_any(p, dtype, i + 2),
                     load_any(p, dtype, i + 3));
}

// Eight rows of y = M x for NV vectors on one warp: lane l reads columns
// 4l .. 4l + 3 of rows row0 .. row0 + 7 (eight coalesced 512-byte row loads)
// against x4[v] = x_v[4l .. 4l + 3]; the per-row partial sums are reduced
// across lanes by three halving exchanges and two full sums, after which
// lane l holds row row0 + rsel(l), rsel(l) = 4 bit4(l) + 2 bit3(l) + bit2(l).
template <int NV>
__device__ __forceinline__ void matvec_rows8(const float* __restrict__ M, int row0, const float4 (&x4)[NV],
                                             float (&y)[NV]) {
  const int lane = threadIdx.x & 31;
  const float4* rows = reinterpret_cast<const float4*>(M + (size_t)row0 * D) + lane;
  float4 t[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) t[i] = __ldg(rows + i * 32);
  float p[NV][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int v = 0; v < NV; ++v)
      p[v][i] = fmaf(t[i].x, x4[v].x, fmaf(t[i].y, x4[v].y, fmaf(t[i].z, x4[v].z, t[i].w * x4[v].w)));
#pragma unroll
  for (int o = 16, n = 4; o >= 4; o >>= 1, n >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int v = 0; v < NV; ++v)
#pragma unroll
      for (int k = 0; k < n; ++k) {
        const float a = p[v][k], b = p[v][k + n];
        p[v][k] = (up ? b : a) + __shfl_xor_sync(FULL, up ? a : b, o);
      }
  }
#pragma unroll
  for (int v = 0; v < NV; ++v) {
    float r = p[v][0];
    r += __shfl_xor_sync(FULL, r, 2);
    r += __shfl_xor_sync(FULL, r, 1);
    y[v] = r;
  }
}

// Query transform of one (sequence b, KV head h) group on a 128-thread CTA:
// q'[g][i] = sum_j M[i][j] q[g][j] for the G query heads of the group, M =
// T_k^{-T} of head h (summary page "WUSH-KV：数据自适应变换的 KV Cache 低比特量化",
// 方法关键点 and 工作参考价值: one d x d product per query; the inverse
// transpose keeps q'.k' = q.k).  Thread i streams row i of M against the G
// query vectors staged in qs ([G][128] floats of shared memory).

template <int G>
__device__ __forceinline__ void query_transform_unit(const void* q, int dtype, const float* TinvT, float* out,
                                                     int b, int h, int n_kv_heads) {
  const int Hq = n_kv_heads * G;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rsel = ((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1);
  float4 x4[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const size_t base = ((size_t)b * Hq + (size_t)h * G + g) * D + 4 * lane;
    x4[g] = make_float4(load_any(q, dtype, base), load_any(q, dtype, base + 1), load_any(q, dtype, base + 2),
                        load_any(q, dtype, base + 3));
  }
#pragma unroll 1
  for (int rg = 0; rg < 4; ++rg) {
    const int row0 = 32 * warp + 8 * rg;
    float y[G];
    matvec_rows8<G>(TinvT + (size_t)h * D * D, row0, x4, y);
    if ((lane & 3) == 0) {
#pragma unroll
      for (int g = 0; g < G; ++g) out[((size_t)b * Hq + (size_t)h * G + g) * D + row0 + rsel] = y[g];
    }
  }
}

// ---------------------------------------------------------------------------
// Per-token quantisers on one warp.  Lane l holds dims 4l..4l+3 of the token
// as float values that are exactly fp16 values.
// ---------------------------------------------------------------------------

// QuEST INT: RMS-based scale, symmetric mid-rise grid, bin-centre
// reconstruction (review "[논문리뷰] WUSH-KV ...", Key Terms, QuEST entry).
// delta = fp16(alpha * rms / 2^(bits-1)); code = clamp(floor(x/delta + L/2)).
__device__ __forceinline__ void quest_warp(const float x[4], int bits, double alpha,
                                           uint8_t code[4], __half& delta) {
  double ss = 0.0;
#pragma unroll
  for (int i = 0; i < 4; ++i) ss = __fma_rn((double)x[i], (double)x[i], ss);
  ss = warp_sum_f64(ss);
  const double rms = __dsqrt_rn(ss / 128.0);
  const double dd = __dmul_rn(alpha, rms) / (double)(1 << (bits - 1));
  delta = f64_to_f16_rn(dd);
  const float d32 = __half2float(delta);
  const int L = 1 << bits;
  const float inv = __frcp_rn(d32);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float t = __fadd_rn(__fmul_rn(x[i], inv), (float)(L / 2));
    t = fminf(fmaxf(floorf(t), 0.f), (float)(L - 1));
    code[i] = (d32 == 0.f) ? (uint8_t)(L / 2) : (uint8_t)(int)t;
  }
}

// k-th smallest (1-indexed, k <= 8) of the warp's 128 values; ties are
// removed one occurrence per round, so the result is the order statistic.
__device__ __forceinline__ float warp_kth_smallest(const float x[4], int k) {
  const int lane = threadIdx.x & 31;
  unsigned taken = 0;
  float m = 0.f;
  for (int round = 0; round < k; ++round) {
    float lm = INFINITY;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (!(taken >> i & 1)) lm = fminf(lm, x[i]);
    float g = lm;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) g = fminf(g, __shfl_xor_sync(FULL, g, o));
    const unsigned who = __ballot_sync(FULL, lm == g);
    if (lane == __ffs(who) - 1) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (!(taken >> i & 1) && x[i] == g) { taken |= 1u << i; break; }
    }
    m = g;
  }
  return m;
}

__device__ __forceinline__ float warp_kth_largest(const float x[4], int k) {
  float y[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) y[i] = -x[i];
  return -warp_kth_smallest(y, k);
}

// Percentile-clipped affine quantiser (summary page 方法关键点, 4th bullet):
// lo/hi = order statistics r_lo, r_hi; s = fp16((hi - lo) / (L - 1));
// code = clamp(rint((x - lo) / s)).  Zeros are canonicalised to +0.
__device__ __forceinline__ void affine_warp(const float x[4], int bits, int r_lo, int r_hi,
                                            uint8_t code[4], __half& s_out, __half& lo_out) {
  const int L = 1 << bits;
  float lo = warp_kth_smallest(x, r_lo);
  float hi = warp_kth_largest(x, 129 - r_hi);
  lo = __fadd_rn(lo, 0.f);
  hi = __fadd_rn(hi, 0.f);
  lo_out = __float2half_rn(lo);
  const float s32 = __fdiv_rn(__fsub_rn(hi, lo), (float)(L - 1));
  s_out = __float2half_rn(s32);
  const float sd = __half2float(s_out);
  const float lo_h = __half2float(lo_out);
  const float inv = __frcp_rn(sd);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float t = __fmul_rn(__fsub_rn(x[i], lo_h), inv);
    t = fminf(fmaxf(rintf(t), 0.f), (float)(L - 1));
    code[i] = (sd == 0.f) ? (uint8_t)0 : (uint8_t)(int)t;
  }
}

// ---------------------------------------------------------------------------
// Packed format index maps (see the layout comment in wushkv.h)
// ---------------------------------------------------------------------------

// K row: dim of field s, byte beta of word wi in a plane of width w.
__device__ __forceinline__ int k_field_dim(int wi, int w, int s, int beta) {
  const int P = 8 / w;
  const int c = wi / w, sub = wi % w;
  const int rho = sub * P + s;
  const int h = rho >> 2, ks = rho & 3;
  return 32 * ks + 4 * c + 16 * h + beta;
}

// V quad: dim of field s, byte beta (token) of word wi (= r*2w + j).
__device__ __forceinline__ int v_field_dim(int wi, int w, int s) {
  const int P = 8 / w;
  const int r = wi / (2 * w), j = wi % (2 * w);
  const int rho = j * P + s;
  const int mt = rho >> 1, rh = rho & 1;
  return 16 * mt + r + 8 * rh;
}

// Flat word index in a V quad of unit word j of row unit r (plane width w):
// the 2w words of row r sit at unit position (r + 2 (quad mod 4)) mod 8; a
// 4-bit unit is split into two 16-byte halves 128 bytes apart.
__host__ __device__ __forceinline__ int v_word_index(int quad, int r, int j, int w) {
  const int pos = (r + 2 * (quad & 3)) & 7;
  if (w == 4) return j < 4 ? 4 * pos + j : 32 + 4 * pos + (j - 4);
  return 2 * w * pos + j;
}

// Value of plane p (width w) of a code: 3-bit codes split into a 2-bit low
// plane and a 1-bit high plane.
__device__ __forceinline__ uint32_t plane_value(uint32_t code, int bits, int p) {
  if (bits == 3) return p == 0 ? (code & 3u) : (code >> 2);
  return code;
}

// ---------------------------------------------------------------------------
// Host-side launchers (defined in the .cu files)
// ---------------------------------------------------------------------------
struct AppendArgs {
  DevCache c;
  const void* k;           // [B][n_tok][Hkv][128]
  const void* v;
  int dtype;
  const float* T;          // [Hkv][128][128] or null
  int n_tok;
  int64_t n0;              // tokens before this append
  int64_t packed0, packed1;  // packed counts before / after
  int64_t quad_begin;      // first absolute quad (4 tokens) handled
  int64_t n_quads;         // quads handled by this launch
  int quads_per_cta;
};
cudaError_t launch_append(const AppendArgs& a, cudaStream_t s);
// A one-token decode-step append whose new token stays in the fp16 windows,
// fused with the step's query transform: per unit, four CTAs for the key
// rows, four for the query rows, and n_flush_quads append CTAs for the quads
// of the chunk this step flushes (a.quad_begin, no transform).
cudaError_t launch_step_rows(const AppendArgs& a, int n_flush_quads, const void* q, int q_dtype,
                             const float* TinvT, float* q_out, cudaStream_t s);
// The append launch of a (single-phase, FMA-path) decode-step append fused
// with the query transform of the step (q_out = T_k^{-T} q per query head).
cudaError_t launch_append_qt(const AppendArgs& a, const void* q, int q_dtype, const float* TinvT,
                             float* q_out, cudaStream_t s);

// Bulk append on the tensor cores: every token t in [ta, tb) of every unit
// comes straight from the bf16 input (keys through T) and goes to the fp16
// sink (t < sink), the packed cache (sink <= t < sink + packed1) or the
// fp16 recent ring.
struct PrefillArgs {
  DevCache c;
  const float* T;          // [Hkv][128][128] fp32, 16-byte aligned
  int n_tok;               // tokens per sequence in this append
  int64_t n0;              // tokens before this append
  int ta, tb;              // absolute token range (ta a multiple of 4, tb = n0 + n_tok)
  int packed1;             // packed count after this append
  int tiles_per_unit;      // ceil((tb - ta) / 128)
  int ctas_per_head;       // CTAs sharing one KV head's tiles
};
cudaError_t launch_prefill_tc(const PrefillArgs& a, const void* k, const void* v, int sms,
                              cudaStream_t s);
// The value rows of the same packed index range (called by launch_prefill_tc).
cudaError_t launch_value_pack(const PrefillArgs& a, const void* v, int sms, cudaStream_t s);

cudaError_t launch_query_transform(const void* q, int dtype, const float* TinvT, float* out,
                                   int batch, int n_q_heads, int n_kv_heads, cudaStream_t s);

// Tensor maps over the fp16 windows (sink and recent ring, K and V), each a
// [units * slots][128] array read in boxes of WIN_BOX_ROWS rows x 64 dims
// with the 128-byte swizzle.  Built once per cache; a region whose map
// could not be built (no sink, or more than 2^31 rows) is read without one.
constexpr int WIN_BOX_ROWS = 8;
struct WindowMaps {
  CUtensorMap sink_k, sink_v, ring_k, ring_v;
  int has_sink, has_ring;
};
void make_window_maps(const DevCache& c, WindowMaps* m);

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
// cuTensorMapEncodeTiled through the runtime's entry-point query (null if absent).
EncodeTiledFn tensor_map_encoder();

struct DecodeArgs {
  DevCache c;
  const float* q;          // [B][Hq][128] fp32
  float* out;              // [B][Hq][128] fp32
  float scale_log2;        // scale * log2(e)
  int n_sink, n_packed, n_recent;
  int ring_first;          // ring slot of the oldest recent token
  int grid;                // CTAs (stream-K shares of the units' items)
  int win_chunks;          // ceil((n_sink + n_recent) / 8)
  int pack_blocks;         // ceil(n_packed / 64)
  int items_per_unit;      // win_chunks + pack_blocks
  uint32_t cta_q, cta_r;   // stream-K split: CTA i starts at item i cta_q + min(i, cta_r)
  float* partials;         // split partials [unit][max_splits][G][132]
  int* counters;           // arrival counter per unit
  uint32_t inject_polls;   // 0, or fault injection for tests: each warp's first copy wait is made on a
                           // barrier nothing completes and gives up after this many polls
};
// Sequences of unequal lengths: each sequence's token count and the first
// global item of its units (items laid end to end, unit by unit); a
// kernel parameter of the decode, so the CTAs find their units without a
// memory round trip.
constexpr int MAX_RAGGED_SEQS = 1024;
struct RaggedTable {
  uint32_t item_start[MAX_RAGGED_SEQS + 1];   // [nseq] = total items
  int32_t n[MAX_RAGGED_SEQS];
  int32_t nseq;
};
// rt: null when every sequence holds the same number of tokens.
cudaError_t launch_decode(const DecodeArgs& a, const WindowMaps& m, const RaggedTable* rt, cudaStream_t s);
int decode_ctas_per_sm(int bits, int group, int quantizer);

// Chunked-prefill attention: q [batch][n_q][n_q_heads][128] fp32 (the last
// n_q tokens' transformed queries), out likewise; every sequence holds n
// tokens (ns sink, P packed, the rest in the ring).
struct PaArgs {
  DevCache c;
  const float* q;
  float* out;
  int n, n_q, ns, P;
  float scale_log2;
};
cudaError_t launch_prefill_attention(const PaArgs& a, cudaStream_t s);

}  // namespace wushkv
