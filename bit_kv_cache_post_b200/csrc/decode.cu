// GQA decode attention over the packed cache plus the fp16 windows, split-K
// over the context with the split partials merged by the last CTA of each
// unit to finish (an arrival counter; no CTA ever waits on another).
//
// Method source: review "[논문리뷰] WUSH-KV ..." (secrett2633), Key Terms
// (GQA: several query heads share one KV head); summary page 动机 and the
// abstract on weekinpapers.com (decode cost is KV memory and bandwidth).
// Dequantisation is fused into the score and PV loops.
#include "wushkv_internal.cuh"

namespace wushkv {

namespace {


// Lane l gets dims 4l..4l+3 of packed key pk of unit u, dequantised.
__device__ __forceinline__ void packed_key(const DevCache& c, int u, int pk, int lane, float k[4]) {
  const int c4 = lane & 3, hh = (lane >> 2) & 1, ks = lane >> 3;
  const int rho = 4 * hh + ks;
  uint32_t code[4] = {0u, 0u, 0u, 0u};
  int shift = 0;
  for (int p = 0; p < c.n_planes; ++p) {
    const int w = c.plane_bits[p], P = 8 / w;
    const uint32_t mask = (1u << w) - 1u;
    const uint32_t* row = reinterpret_cast<const uint32_t*>(
        c.k_plane[p] + (size_t)u * c.plane_unit_stride[p] + (size_t)pk * 16 * w);
    const uint32_t wd = row[c4 * w + rho / P];
    const int s = rho % P;
#pragma unroll
    for (int beta = 0; beta < 4; ++beta) code[beta] |= ((wd >> (8 * beta + w * s)) & mask) << shift;
    shift += w;
  }
  const uint8_t* meta = c.k_meta + (size_t)u * c.meta_unit_stride + (size_t)pk * c.meta_bytes;
  if (c.quantizer == WUSHKV_QUEST_INT) {
    const float dl = __half2float(*reinterpret_cast<const __half*>(meta));
    const float off = 0.5f - (float)(1 << (c.bits - 1));
#pragma unroll
    for (int i = 0; i < 4; ++i) k[i] = ((float)code[i] + off) * dl;
  } else {
    const __half2 sl = *reinterpret_cast<const __half2*>(meta);
    const float s = __low2float(sl), lo = __high2float(sl);
#pragma unroll
    for (int i = 0; i < 4; ++i) k[i] = fmaf((float)code[i], s, lo);
  }
}

// Lane l gets dims 4l..4l+3 of packed value pk of unit u, dequantised.
__device__ __forceinline__ void packed_value(const DevCache& c, int u, int pk, int lane, float v[4]) {
  const int mt = lane >> 2, rh = (lane >> 1) & 1;
  const int rho = 2 * mt + rh;
  const int beta = pk & 3;
  uint32_t code[4] = {0u, 0u, 0u, 0u};
  int shift = 0;
  for (int p = 0; p < c.n_planes; ++p) {
    const int w = c.plane_bits[p], P = 8 / w;
    const uint32_t mask = (1u << w) - 1u;
    const uint32_t* quad = reinterpret_cast<const uint32_t*>(
        c.v_plane[p] + (size_t)u * c.plane_unit_stride[p] + (size_t)(pk >> 2) * 64 * w);
    const int s = rho % P;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = 4 * (lane & 1) + i;
      const uint32_t wd = quad[r * 2 * w + rho / P];
      code[i] |= ((wd >> (8 * beta + w * s)) & mask) << shift;
    }
    shift += w;
  }
  const uint8_t* meta = c.v_meta + (size_t)u * c.meta_unit_stride + (size_t)pk * c.meta_bytes;
  if (c.quantizer == WUSHKV_QUEST_INT) {
    const float dl = __half2float(*reinterpret_cast<const __half*>(meta));
    const float off = 0.5f - (float)(1 << (c.bits - 1));
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = ((float)code[i] + off) * dl;
  } else {
    const __half2 sl = *reinterpret_cast<const __half2*>(meta);
    const float s = __low2float(sl), lo = __high2float(sl);
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = fmaf((float)code[i], s, lo);
  }
}

__device__ __forceinline__ void load_row4(const __half* row, int lane, float x[4]) {
  const uint2 raw = *reinterpret_cast<const uint2*>(row + 4 * lane);
  const __half2 a = *reinterpret_cast<const __half2*>(&raw.x);
  const __half2 b = *reinterpret_cast<const __half2*>(&raw.y);
  x[0] = __low2float(a); x[1] = __high2float(a);
  x[2] = __low2float(b); x[3] = __high2float(b);
}

// Merge (m, l, o) partials: weights exp2(m_i - M); empty partials (m = -inf)
// weigh zero.
__device__ __forceinline__ float merge_weight(float m, float M) {
  return (m == -INFINITY) ? 0.f : exp2f(m - M);
}

template <int G>
__global__ void __launch_bounds__(128) decode_simt_kernel(DecodeArgs a) {
  const DevCache& c = a.c;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int u = blockIdx.y, split = blockIdx.x;
  const int b = u / c.n_kv_heads, h = u % c.n_kv_heads;
  const int Hq = c.n_kv_heads * G;
  const int total_splits = a.win_splits + a.pack_splits;

  __shared__ float qs[G][D];
  __shared__ float wm[4][G], wl[4][G];
  __shared__ float wo[4][G][D];
  __shared__ int is_last;

  for (int g = 0; g < G; ++g)
    qs[g][tid] = a.q[((size_t)b * Hq + (size_t)h * G + g) * D + tid] * a.scale_log2;
  __syncthreads();

  const bool window = split < a.win_splits;
  int t0, t1;
  if (window) {
    t0 = split * a.win_tokens_per_split;
    t1 = min(t0 + a.win_tokens_per_split, a.n_sink + a.n_recent);
  } else {
    t0 = (split - a.win_splits) * a.pack_tokens_per_split;
    t1 = min(t0 + a.pack_tokens_per_split, a.n_packed);
  }

  float m[G], l[G], o[G][4];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY; l[g] = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) o[g][i] = 0.f;
  }

  for (int t = t0 + warp; t < t1; t += 4) {
    float kk[4], vv[4];
    if (window) {
      const __half *kr, *vr;
      if (t < a.n_sink) {
        const size_t off = ((size_t)u * c.sink + t) * D;
        kr = c.sink_k + off; vr = c.sink_v + off;
      } else {
        const int slot = (a.ring_first + (t - a.n_sink)) % c.ring_slots;
        const size_t off = ((size_t)u * c.ring_slots + slot) * D;
        kr = c.ring_k + off; vr = c.ring_v + off;
      }
      load_row4(kr, lane, kk);
      load_row4(vr, lane, vv);
    } else {
      packed_key(c, u, t, lane, kk);
      packed_value(c, u, t, lane, vv);
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float s = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) s = fmaf(qs[g][4 * lane + i], kk[i], s);
      s = warp_sum_f32(s);
      const float mn = fmaxf(m[g], s);
      const float al = exp2f(m[g] - mn);
      const float p = exp2f(s - mn);
      l[g] = fmaf(l[g], al, p);
#pragma unroll
      for (int i = 0; i < 4; ++i) o[g][i] = fmaf(o[g][i], al, p * vv[i]);
      m[g] = mn;
    }
  }

#pragma unroll
  for (int g = 0; g < G; ++g) {
    if (lane == 0) { wm[warp][g] = m[g]; wl[warp][g] = l[g]; }
#pragma unroll
    for (int i = 0; i < 4; ++i) wo[warp][g][4 * lane + i] = o[g][i];
  }
  __syncthreads();

  float* part_base = a.partials + ((size_t)u * c.max_splits + split) * G * (D + 2);
  for (int g = 0; g < G; ++g) {
    float M = -INFINITY;
    for (int w = 0; w < 4; ++w) M = fmaxf(M, wm[w][g]);
    float L = 0.f, O = 0.f;
    for (int w = 0; w < 4; ++w) {
      const float f = merge_weight(wm[w][g], M);
      L = fmaf(wl[w][g], f, L);
      O = fmaf(wo[w][g][tid], f, O);
    }
    float* part = part_base + (size_t)g * (D + 2);
    part[tid] = O;
    if (tid == 0) { part[D] = M; part[D + 1] = L; }
  }

  // Arrival: the last CTA of this unit merges every split.
  __threadfence();
  __syncthreads();
  if (tid == 0) is_last = (atomicAdd(a.counters + u, 1) == total_splits - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  for (int g = 0; g < G; ++g) {
    float M = -INFINITY;
    for (int sp = 0; sp < total_splits; ++sp) {
      const float* part = a.partials + (((size_t)u * c.max_splits + sp) * G + g) * (D + 2);
      M = fmaxf(M, __ldcg(part + D));
    }
    float L = 0.f, O = 0.f;
    for (int sp = 0; sp < total_splits; ++sp) {
      const float* part = a.partials + (((size_t)u * c.max_splits + sp) * G + g) * (D + 2);
      const float f = merge_weight(__ldcg(part + D), M);
      L = fmaf(__ldcg(part + D + 1), f, L);
      O = fmaf(__ldcg(part + tid), f, O);
    }
    a.out[((size_t)b * Hq + (size_t)h * G + g) * D + tid] = O / L;
  }
  if (tid == 0) a.counters[u] = 0;
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s) {
  const int total = a.win_splits + a.pack_splits;
  dim3 grid((unsigned)total, (unsigned)a.c.units);
  switch (a.c.group) {
    case 1: decode_simt_kernel<1><<<grid, 128, 0, s>>>(a); break;
    case 2: decode_simt_kernel<2><<<grid, 128, 0, s>>>(a); break;
    case 4: decode_simt_kernel<4><<<grid, 128, 0, s>>>(a); break;
    case 8: decode_simt_kernel<8><<<grid, 128, 0, s>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace wushkv
