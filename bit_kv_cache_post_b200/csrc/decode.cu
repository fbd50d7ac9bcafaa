// GQA decode attention over the packed cache plus the fp16 windows.
//
// Method source: review "[논문리뷰] WUSH-KV ..." (secrett2633), Key Terms (GQA:
// several query heads share one KV head); summary page 动机 and the abstract
// on weekinpapers.com (decode cost is KV memory and bandwidth).
// Dequantisation is fused into the score and PV loops:
//   score(t) = scale_t * (q' . c_t) + offset_t * sum(q')
//   out      = sum_t p_t scale_t c_t + sum_t p_t offset_t      (then / sum p)
// with (scale, offset) = (delta, delta (1/2 - L/2)) for QuEST INT and
// (s, lo) for the affine quantiser.
//
// Work split: each unit (sequence, KV head) is cut into `splits` CTAs of
// equal bytes (32-token groups of the fp16 windows, 64-token blocks of the
// packed cache); the grid is one wave.  Inside a CTA, 4 warps take groups
// and blocks round-robin.  The packed blocks run on integer tensor cores
// (mma.sync m16n8k32): codes (u8) x two int8 terms of the query for the
// scores, codes (u8) x two u8 terms of p * scale for PV.  The window tokens
// run one token per lane in fp32.  Each CTA merges its warps and writes one
// (m, l, o) partial; the last CTA of a unit to finish merges the partials
// (an arrival counter; no CTA ever waits on another).
#include "decode_frag.cuh"

namespace wushkv {

namespace {

constexpr int NW = 4;     // warps per CTA
constexpr int PB = 64;    // packed tokens per warp block
constexpr int WGRP = 32;  // window tokens per warp group
constexpr int PS_LD = PB + 16;  // bytes per row of the per-warp P tile (bank-conflict free)

template <int G>
struct Smem {
  static constexpr int NT = (G + 3) / 4;       // n-tiles of 8 columns (4 heads x 2 terms)
  float qs[G][D];                              // scaled q' (fp32)
  int8_t qterm[NT * 4][2][D];                  // two int8 terms per head (padded heads = 0)
  float qscale[NT * 4];                        // sigma / 254 per head
  float qsum[NT * 4];                          // sum of the quantised q per head
  uint8_t ps[NW][NT * 8][PS_LD];               // per-warp P terms [col][token]
  float sm[2 * NW][G], sl[2 * NW][G];          // per-slot softmax max / sum
  float so[2 * NW][G][D];                      // per-slot unnormalised outputs
  int is_last;
};

__device__ __forceinline__ float merge_weight(float m, float M) {
  return (m == -INFINITY) ? 0.f : exp2f(m - M);
}

__device__ __forceinline__ int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }

// First item (window group or packed block) of split s.
__device__ __forceinline__ int split_begin(const DecodeArgs& a, int s) {
  if (s >= a.splits) return a.win_groups + a.pack_blocks;
  const int64_t wcost = (int64_t)a.win_groups * a.cost_w;
  const int64_t total = wcost + (int64_t)a.pack_blocks * a.cost_p;
  const int64_t x = total * s / a.splits;
  if (x < wcost) return (int)ceil_div64(x, a.cost_w);
  return a.win_groups + (int)ceil_div64(x - wcost, a.cost_p);
}

// ---- fp16 window tokens: one token per lane -----------------------------------
template <int G>
__device__ __forceinline__ const __half* window_row(const DecodeArgs& a, const __half* sink,
                                                    const __half* ring, int u, int w) {
  const DevCache& c = a.c;
  if (w < a.n_sink) return sink + ((size_t)u * c.sink + w) * D;
  const int slot = (a.ring_first + (w - a.n_sink)) % c.ring_slots;
  return ring + ((size_t)u * c.ring_slots + slot) * D;
}

template <int G>
__device__ void window_groups(const DecodeArgs& a, Smem<G>& sh, int u, int g0, int g1, int warp,
                              int lane, int slot) {
  const DevCache& c = a.c;
  float m[G], l[G], o[G][4];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY; l[g] = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) o[g][i] = 0.f;
  }
  for (int grp = g0 + warp; grp < g1; grp += NW) {
    const int w = grp * WGRP + lane;
    const bool valid = w < a.n_sink + a.n_recent;
    float s[G];
#pragma unroll
    for (int g = 0; g < G; ++g) s[g] = 0.f;
    if (valid) {
      const uint4* krow = reinterpret_cast<const uint4*>(window_row<G>(a, c.sink_k, c.ring_k, u, w));
#pragma unroll 4
      for (int ch = 0; ch < D / 8; ++ch) {
        const uint4 raw = __ldg(krow + ch);
        const __half2* h2 = reinterpret_cast<const __half2*>(&raw);
        float x[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __half22float2(h2[i]);
          x[2 * i] = f.x; x[2 * i + 1] = f.y;
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float4 qa = *reinterpret_cast<const float4*>(&sh.qs[g][8 * ch]);
          const float4 qb = *reinterpret_cast<const float4*>(&sh.qs[g][8 * ch + 4]);
          s[g] = fmaf(qa.x, x[0], s[g]); s[g] = fmaf(qa.y, x[1], s[g]);
          s[g] = fmaf(qa.z, x[2], s[g]); s[g] = fmaf(qa.w, x[3], s[g]);
          s[g] = fmaf(qb.x, x[4], s[g]); s[g] = fmaf(qb.y, x[5], s[g]);
          s[g] = fmaf(qb.z, x[6], s[g]); s[g] = fmaf(qb.w, x[7], s[g]);
        }
      }
    }
    float p[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float sv = valid ? s[g] : -INFINITY;
      const float mn = fmaxf(m[g], warp_max_f32(sv));
      const float al = exp2f(m[g] - mn);
      p[g] = valid ? exp2f(sv - mn) : 0.f;
      l[g] = fmaf(l[g], al, p[g]);
#pragma unroll
      for (int i = 0; i < 4; ++i) o[g][i] *= al;
      m[g] = mn;
    }
    const int nvalid = min(WGRP, a.n_sink + a.n_recent - grp * WGRP);
#pragma unroll 4
    for (int j = 0; j < nvalid; ++j) {
      const __half* vrow = window_row<G>(a, c.sink_v, c.ring_v, u, grp * WGRP + j);
      const uint2 raw = __ldg(reinterpret_cast<const uint2*>(vrow) + lane);
      const float2 v01 = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
      const float2 v23 = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float pj = __shfl_sync(FULL, p[g], j);
        o[g][0] = fmaf(pj, v01.x, o[g][0]); o[g][1] = fmaf(pj, v01.y, o[g][1]);
        o[g][2] = fmaf(pj, v23.x, o[g][2]); o[g][3] = fmaf(pj, v23.y, o[g][3]);
      }
    }
  }
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float lt = warp_sum_f32(l[g]);
    if (lane == 0) { sh.sm[slot][g] = m[g]; sh.sl[slot][g] = lt; }
#pragma unroll
    for (int i = 0; i < 4; ++i) sh.so[slot][g][4 * lane + i] = o[g][i];
  }
}

// ---- packed tokens: integer tensor cores ----------------------------------------
// Lane = 4r + c.  Score m-tile rows r, r+8 are tokens; columns are (head,
// term) pairs, so thread c owns head 4nt + c of n-tile nt.  PV m-tile rows
// are dims 16mt + r (+8); the PV B operand comes back through the warp's P
// tile in shared memory.
template <int BITS, int G, bool AFFINE>
__device__ void packed_blocks(const DecodeArgs& a, Smem<G>& sh, int u, int b0, int b1, int warp,
                              int lane, int slot) {
  constexpr int NT = Smem<G>::NT;
  const DevCache& c = a.c;
  const int r = lane >> 2, c4 = lane & 3;
  const float beta = 0.5f - (float)(1 << (BITS - 1));
  const uint8_t* kp0 = c.k_plane[0] + (size_t)u * c.plane_unit_stride[0];
  const uint8_t* kp1 = c.k_plane[1] + (size_t)u * c.plane_unit_stride[1];
  const uint8_t* vp0 = c.v_plane[0] + (size_t)u * c.plane_unit_stride[0];
  const uint8_t* vp1 = c.v_plane[1] + (size_t)u * c.plane_unit_stride[1];
  const uint8_t* kmeta = c.k_meta + (size_t)u * c.meta_unit_stride;
  const uint8_t* vmeta = c.v_meta + (size_t)u * c.meta_unit_stride;

  // B fragments of the quantised query: n-tile nt, k-step ks, half h
  uint32_t qb[NT][4][2];
  float qscale[NT], qsum[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int gcol = nt * 4 + (r >> 1), term = r & 1;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
#pragma unroll
      for (int h = 0; h < 2; ++h)
        qb[nt][ks][h] = *reinterpret_cast<const uint32_t*>(&sh.qterm[gcol][term][32 * ks + 16 * h + 4 * c4]);
    qscale[nt] = sh.qscale[nt * 4 + c4];
    qsum[nt] = sh.qsum[nt * 4 + c4];
  }

  float mP[NT], lP[NT], eP[NT], oP[NT][8][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    mP[nt] = -INFINITY; lP[nt] = 0.f; eP[nt] = 0.f;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) oP[nt][mt][0] = oP[nt][mt][1] = 0.f;
  }
  uint8_t* ps = &sh.ps[warp][0][0];

  for (int blk = b0 + warp; blk < b1; blk += NW) {
    const int tb = blk * PB;
    // ---- loads: K rows, V quads, per-token scales -----------------------------
    KWords<BITS> kw[4][2];
    float2 km[4][2], vm[4][2];
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int th = 0; th < 2; ++th) {
        const int tok = tb + 16 * mt + r + 8 * th;
        kw[mt][th] = load_k_words<BITS>(kp0, kp1, tok, c4);
        km[mt][th] = load_meta<AFFINE>(kmeta, tok, beta);
        vm[mt][th] = load_meta<AFFINE>(vmeta, tok, beta);
      }
    VWords<BITS> vw[2][2];
#pragma unroll
    for (int k2 = 0; k2 < 2; ++k2)
#pragma unroll
      for (int q = 0; q < 2; ++q)
        vw[k2][q] = load_v_words<BITS>(vp0, vp1, (tb + 32 * k2) / 4 + c4 + 4 * q, r);

    // ---- scores ----------------------------------------------------------------
    float sc[4][2][NT];
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      int acc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0;
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const uint32_t a0 = k_frag<BITS>(kw[mt][0], ks, 0), a1 = k_frag<BITS>(kw[mt][1], ks, 0);
        const uint32_t a2 = k_frag<BITS>(kw[mt][0], ks, 1), a3 = k_frag<BITS>(kw[mt][1], ks, 1);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_u8s8(acc[nt], a0, a1, a2, a3, qb[nt][ks][0], qb[nt][ks][1]);
      }
#pragma unroll
      for (int th = 0; th < 2; ++th) {
        const bool valid = tb + 16 * mt + r + 8 * th < a.n_packed;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const float dot = qscale[nt] * (float)(acc[nt][2 * th] * 254 + acc[nt][2 * th + 1]);
          const float s = fmaf(km[mt][th].x, dot, km[mt][th].y * qsum[nt]);
          sc[mt][th][nt] = valid ? s : -INFINITY;
        }
      }
    }

    // ---- online softmax, P terms -------------------------------------------------
    float al[NT], sp[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float bm = -INFINITY;
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) bm = fmaxf(bm, fmaxf(sc[mt][0][nt], sc[mt][1][nt]));
      bm = fmaxf(bm, __shfl_xor_sync(FULL, bm, 4));
      bm = fmaxf(bm, __shfl_xor_sync(FULL, bm, 8));
      bm = fmaxf(bm, __shfl_xor_sync(FULL, bm, 16));
      const float mn = fmaxf(mP[nt], bm);
      al[nt] = exp2f(mP[nt] - mn);
      mP[nt] = mn;
      float ls = 0.f, es = 0.f, pm = 0.f;
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int th = 0; th < 2; ++th) {
          const float p = exp2f(sc[mt][th][nt] - mn);
          const bool valid = sc[mt][th][nt] != -INFINITY;
          const float pt = valid ? p * vm[mt][th].x : 0.f;
          ls += p;
          es = valid ? fmaf(p, vm[mt][th].y, es) : es;
          pm = fmaxf(pm, pt);
          sc[mt][th][nt] = pt;
        }
      pm = fmaxf(pm, __shfl_xor_sync(FULL, pm, 4));
      pm = fmaxf(pm, __shfl_xor_sync(FULL, pm, 8));
      pm = fmaxf(pm, __shfl_xor_sync(FULL, pm, 16));
      sp[nt] = pm;
      lP[nt] = fmaf(lP[nt], al[nt], ls);
      eP[nt] = fmaf(eP[nt], al[nt], es);
      const float inv = pm > 0.f ? 255.f / pm : 0.f;
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int th = 0; th < 2; ++th) {
          const float uu = fminf(sc[mt][th][nt] * inv, 255.f);
          const float q0 = floorf(uu);
          const float q1 = fminf(rintf((uu - q0) * 255.f), 255.f);
          const int col = nt * 8 + 2 * c4;
          const int t = 16 * mt + r + 8 * th;
          ps[col * PS_LD + t] = (uint8_t)q0;
          ps[(col + 1) * PS_LD + t] = (uint8_t)q1;
        }
    }
    __syncwarp();

    // ---- PV: dims x (head, term) over 64 tokens ----------------------------------
    int pacc[8][NT][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) pacc[mt][nt][0] = pacc[mt][nt][1] = pacc[mt][nt][2] = pacc[mt][nt][3] = 0;
#pragma unroll
    for (int k2 = 0; k2 < 2; ++k2) {
      uint32_t pb[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const uint8_t* row = ps + (nt * 8 + r) * PS_LD + 32 * k2 + 4 * c4;
        pb[nt][0] = *reinterpret_cast<const uint32_t*>(row);
        pb[nt][1] = *reinterpret_cast<const uint32_t*>(row + 16);
      }
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        const uint32_t a0 = v_frag<BITS>(vw[k2][0], 2 * mt), a1 = v_frag<BITS>(vw[k2][0], 2 * mt + 1);
        const uint32_t a2 = v_frag<BITS>(vw[k2][1], 2 * mt), a3 = v_frag<BITS>(vw[k2][1], 2 * mt + 1);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_u8u8(pacc[mt][nt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
      }
    }
    __syncwarp();
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const float f = sp[nt] * (1.f / 65025.f);
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        oP[nt][mt][0] = fmaf(oP[nt][mt][0], al[nt], f * (float)(pacc[mt][nt][0] * 255 + pacc[mt][nt][1]));
        oP[nt][mt][1] = fmaf(oP[nt][mt][1], al[nt], f * (float)(pacc[mt][nt][2] * 255 + pacc[mt][nt][3]));
      }
    }
  }

  // ---- warp partial: reduce l, e over the 8 lanes that share a head ----------
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float lt = lP[nt], et = eP[nt];
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      lt += __shfl_xor_sync(FULL, lt, o);
      et += __shfl_xor_sync(FULL, et, o);
    }
    const int g = nt * 4 + c4;
    if (g < G) {
      if (r == 0) { sh.sm[slot][g] = mP[nt]; sh.sl[slot][g] = lt; }
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        sh.so[slot][g][16 * mt + r] = oP[nt][mt][0] + et;
        sh.so[slot][g][16 * mt + r + 8] = oP[nt][mt][1] + et;
      }
    }
  }
}

// ---- the kernel --------------------------------------------------------------------
template <int BITS, int G, bool AFFINE>
__global__ void __launch_bounds__(NW * 32) decode_kernel(DecodeArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Smem<G>& sh = *reinterpret_cast<Smem<G>*>(smem_raw);
  constexpr int NT = Smem<G>::NT;
  const DevCache& c = a.c;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int u = blockIdx.x / a.splits, split = blockIdx.x % a.splits;
  const int b = u / c.n_kv_heads, h = u % c.n_kv_heads;
  const int Hq = c.n_kv_heads * G;

  // ---- scaled query and its two int8 terms per head --------------------------
  for (int g = 0; g < G; ++g)
    sh.qs[g][tid] = a.q[((size_t)b * Hq + (size_t)h * G + g) * D + tid] * a.scale_log2;
  __syncthreads();
  for (int g = warp; g < NT * 4; g += NW) {
    float x[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = g < G ? sh.qs[g][4 * lane + i] : 0.f;
    float mx = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
    mx = warp_max_f32(mx);
    const float sigma = mx / 127.f;
    const float inv = mx > 0.f ? 127.f / mx : 0.f;
    int sum = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float y = x[i] * inv;
      const float t0 = fminf(fmaxf(rintf(y), -127.f), 127.f);
      const float t1 = fminf(fmaxf(rintf((y - t0) * 254.f), -127.f), 127.f);
      sh.qterm[g][0][4 * lane + i] = (int8_t)t0;
      sh.qterm[g][1][4 * lane + i] = (int8_t)t1;
      sum += (int)t0 * 254 + (int)t1;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(FULL, sum, o);
    if (lane == 0) {
      sh.qscale[g] = sigma / 254.f;
      sh.qsum[g] = (sigma / 254.f) * (float)sum;
    }
  }
  __syncthreads();

  // ---- this split's window groups and packed blocks ---------------------------------
  const int i0 = split_begin(a, split), i1 = split_begin(a, split + 1);
  const int wg0 = min(i0, a.win_groups), wg1 = min(i1, a.win_groups);
  const int pb0 = max(i0, a.win_groups) - a.win_groups, pb1 = max(i1, a.win_groups) - a.win_groups;
  // window part: slots 0..NW-1, packed part: slots NW..2NW-1; the packed
  // blocks start on the warp after the last window group
  window_groups<G>(a, sh, u, wg0, wg1, warp, lane, warp);
  const int rot = (wg1 - wg0) % NW;
  const int pwarp = (warp - rot + NW) % NW;
  packed_blocks<BITS, G, AFFINE>(a, sh, u, pb0, pb1, pwarp, lane, NW + warp);
  __syncthreads();

  // ---- merge the 2 NW slots, write this split's partial ------------------------------
  float* part_base = a.partials + ((size_t)u * c.max_splits + split) * G * (D + 2);
  for (int g = 0; g < G; ++g) {
    float M = -INFINITY;
    for (int s = 0; s < 2 * NW; ++s) M = fmaxf(M, sh.sm[s][g]);
    float L = 0.f, O = 0.f;
    for (int s = 0; s < 2 * NW; ++s) {
      const float f = merge_weight(sh.sm[s][g], M);
      L = fmaf(sh.sl[s][g], f, L);
      O = fmaf(sh.so[s][g][tid], f, O);
    }
    float* part = part_base + (size_t)g * (D + 2);
    part[tid] = O;
    if (tid == 0) { part[D] = M; part[D + 1] = L; }
  }

  // ---- arrival: the last CTA of the unit merges every split ----------------------
  __threadfence();
  __syncthreads();
  if (tid == 0) sh.is_last = (atomicAdd(a.counters + u, 1) == a.splits - 1);
  __syncthreads();
  if (!sh.is_last) return;
  __threadfence();
  for (int g = 0; g < G; ++g) {
    float M = -INFINITY;
    for (int sp = 0; sp < a.splits; ++sp)
      M = fmaxf(M, __ldcg(a.partials + (((size_t)u * c.max_splits + sp) * G + g) * (D + 2) + D));
    float L = 0.f, O = 0.f;
    for (int sp = 0; sp < a.splits; ++sp) {
      const float* part = a.partials + (((size_t)u * c.max_splits + sp) * G + g) * (D + 2);
      const float f = merge_weight(__ldcg(part + D), M);
      L = fmaf(__ldcg(part + D + 1), f, L);
      O = fmaf(__ldcg(part + tid), f, O);
    }
    a.out[((size_t)b * Hq + (size_t)h * G + g) * D + tid] = O / L;
  }
  if (tid == 0) a.counters[u] = 0;
}

template <int BITS, int G, bool AFFINE>
cudaError_t launch_t(const DecodeArgs& a, cudaStream_t s) {
  auto k = decode_kernel<BITS, G, AFFINE>;
  const int smem = (int)sizeof(Smem<G>);
  static int attr_done[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr_done[dev] = 1;
  }
  k<<<(unsigned)(a.c.units * a.splits), NW * 32, smem, s>>>(a);
  return cudaGetLastError();
}

template <int BITS, bool AFFINE>
cudaError_t launch_g(const DecodeArgs& a, cudaStream_t s) {
  switch (a.c.group) {
    case 1: return launch_t<BITS, 1, AFFINE>(a, s);
    case 2: return launch_t<BITS, 2, AFFINE>(a, s);
    case 4: return launch_t<BITS, 4, AFFINE>(a, s);
    case 8: return launch_t<BITS, 8, AFFINE>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

template <int BITS, int G, bool AFFINE>
int occupancy_t() {
  int n = 0;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_kernel<BITS, G, AFFINE>, NW * 32,
                                                sizeof(Smem<G>));
  return n;
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s) {
  const bool affine = a.c.quantizer == WUSHKV_AFFINE_PCTCLIP;
  switch (a.c.bits) {
    case 2: return affine ? launch_g<2, true>(a, s) : launch_g<2, false>(a, s);
    case 3: return affine ? launch_g<3, true>(a, s) : launch_g<3, false>(a, s);
    case 4: return affine ? launch_g<4, true>(a, s) : launch_g<4, false>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

// Resident CTAs per SM of the decode kernel for this configuration (the
// split policy fills one wave).
int decode_ctas_per_sm(int bits, int group, int quantizer) {
  const bool af = quantizer == WUSHKV_AFFINE_PCTCLIP;
#define WUSHKV_OCC(B, G) (af ? occupancy_t<B, G, true>() : occupancy_t<B, G, false>())
#define WUSHKV_OCC_G(B)                                              \
  (group == 1 ? WUSHKV_OCC(B, 1) : group == 2 ? WUSHKV_OCC(B, 2)     \
   : group == 4 ? WUSHKV_OCC(B, 4) : WUSHKV_OCC(B, 8))
  if (bits == 2) return WUSHKV_OCC_G(2);
  if (bits == 3) return WUSHKV_OCC_G(3);
  return WUSHKV_OCC_G(4);
#undef WUSHKV_OCC_G
#undef WUSHKV_OCC
}

}  // namespace wushkv
