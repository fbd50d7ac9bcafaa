// Bulk (prefill) append of values: the value rows of one append from its
// first quad boundary on (the token range of the tensor-core key kernel),
// each to the fp16 sink, the packed cache or the fp16 recent ring.
//
// Method source: summary page "WUSH-KV：数据自适应变换的 KV Cache 低比特量化"
// (ai-papers-daily), sections 工作参考价值 and 方法关键点: values need no
// transform (T_V is folded into W_V / W_O); every token vector leaving the
// fp16 recent window is quantised per token and bit-packed.
//
// A warp takes one quad of 4 tokens x 4 consecutive KV heads of one
// sequence, two lanes per row: lane = 8 * token + 2 * head + half, each lane
// holding 64 of the 128 dims (so the four tokens of a quad are lanes 8
// apart and the warp's rows are 1 KB runs of the [B][n_tok][Hkv][128]
// input).  Each lane loads its half row and rounds it to fp16.  A quad
// inside the packed range (its boundaries are multiples of 4) is quantised:
// per-token parameters merged across the row's two lanes, then each lane's
// bytes of its half of the quad words, completed by byte transposes among
// the quad's lanes; any other quad stores its fp16 rows to the sink or ring.
#include "wushkv_internal.cuh"
#include "quant_row.cuh"

namespace wushkv {

namespace {

using namespace rowq;

constexpr int VP_WARPS = 4;

template <int BITS, bool AFFINE>
__global__ void __launch_bounds__(VP_WARPS * 32) value_pack_kernel(const PrefillArgs a,
                                                                   const __nv_bfloat16* v,
                                                                   int64_t n_items, int quads) {
  const DevCache& c = a.c;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t item = (int64_t)blockIdx.x * VP_WARPS + warp;
  if (item >= n_items) return;                       // uniform per warp
  const int Hkv = c.n_kv_heads;
  const int n_hg = (Hkv + 3) >> 2;
  const int hg = (int)(item % n_hg);
  const int64_t rest = item / n_hg;
  const int qi = (int)(rest % quads);
  const int b = (int)(rest / quads);
  const int beta = lane >> 3, hf = lane & 1, h = hg * 4 + ((lane >> 1) & 3);
  const int tq = a.ta + 4 * qi;                      // absolute token of the quad
  const int tok_abs = tq + beta;
  const bool valid = h < Hkv && tok_abs < a.tb;
  const int64_t tok = tok_abs - a.n0;                // token index within this append
  const int pkq = tq - c.sink;
  const bool packed_quad = tq >= c.sink && pkq < a.packed1;   // uniform per warp
  const int pk = pkq + beta;
  // (lanes past the last head write nothing; their addresses are those of a
  // real unit, so no lookup leaves the sequence's page-table row)
  const int u = b * Hkv + min(h, Hkv - 1);
  const uint4* src =
      reinterpret_cast<const uint4*>(v + (((int64_t)b * a.n_tok + tok) * Hkv + h) * D + 64 * hf);
  if (!packed_quad) {
    // fp16 sink or ring row (no quantisation, no lane exchange)
    if (valid) {
      __half* dst = tok_abs < c.sink
                        ? c.sink_v + ((size_t)u * c.sink + tok_abs) * D
                        : c.ring_v + ((size_t)u * c.ring_slots + (size_t)(pk % c.ring_slots)) * D;
      uint4* o = reinterpret_cast<uint4*>(dst + 64 * hf);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint4 rw = __ldg(src + i);
        const __half2 h0 = bf16x2_to_h2(rw.x), h1 = bf16x2_to_h2(rw.y);
        const __half2 h2 = bf16x2_to_h2(rw.z), h3 = bf16x2_to_h2(rw.w);
        o[i] = make_uint4(*reinterpret_cast<const uint32_t*>(&h0), *reinterpret_cast<const uint32_t*>(&h1),
                          *reinterpret_cast<const uint32_t*>(&h2), *reinterpret_cast<const uint32_t*>(&h3));
      }
    }
    return;
  }
  __half2 xh[32];
  {
    uint4 raw[8];
    if (valid) {
#pragma unroll
      for (int i = 0; i < 8; ++i) raw[i] = __ldg(src + i);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) raw[i] = make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      xh[4 * i] = bf16x2_to_h2(raw[i].x);
      xh[4 * i + 1] = bf16x2_to_h2(raw[i].y);
      xh[4 * i + 2] = bf16x2_to_h2(raw[i].z);
      xh[4 * i + 3] = bf16x2_to_h2(raw[i].w);
    }
  }
  QParams q;
  if constexpr (AFFINE) {
    AffineStats st;
    st.init();
#pragma unroll
    for (int e = 0; e < 16; ++e) st.add2(xh[2 * e], xh[2 * e + 1]);
    affine_merge_pair(st);
    affine_finish(st, BITS, c.r_lo == 2, c.r_hi == 127, q);
  } else {
    QuestStats st;
    st.init();
#pragma unroll
    for (int e = 0; e < 32; ++e) st.add(xh[e]);
    quest_merge_pair(st);
    quest_finish(st, BITS, c.alpha, q);
  }
  const int quad = pkq >> 2;
  emit_v_quad_half<BITS, AFFINE, 8>(
      xh, q, beta, hf, quad, v_quad_at(c, 0, u, quad), BITS == 3 ? v_quad_at(c, 1, u, quad) : nullptr,
      valid);
  if (valid && hf == 0) {
    uint8_t* meta = v_meta_at(c, u, pk);
    if constexpr (AFFINE) *reinterpret_cast<uint32_t*>(meta) = q.meta;
    else *reinterpret_cast<uint16_t*>(meta) = (uint16_t)q.meta;
  }
}

template <int BITS, bool AFFINE>
cudaError_t launch_vt(const PrefillArgs& a, const void* v, int64_t n_items, int quads,
                      cudaStream_t s) {
  const int64_t blocks = (n_items + VP_WARPS - 1) / VP_WARPS;
  value_pack_kernel<BITS, AFFINE><<<(unsigned)blocks, VP_WARPS * 32, 0, s>>>(
      a, static_cast<const __nv_bfloat16*>(v), n_items, quads);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_value_pack(const PrefillArgs& a, const void* v, int sms, cudaStream_t s) {
  (void)sms;
  const int B = a.c.units / a.c.n_kv_heads;
  const int quads = (a.tb - a.ta + 3) / 4;
  const int64_t n_items = (int64_t)B * quads * ((a.c.n_kv_heads + 3) / 4);
  if (n_items <= 0) return cudaSuccess;
  const bool aff = a.c.quantizer == WUSHKV_AFFINE_PCTCLIP;
  switch (a.c.bits) {
    case 2: return aff ? launch_vt<2, true>(a, v, n_items, quads, s) : launch_vt<2, false>(a, v, n_items, quads, s);
    case 3: return aff ? launch_vt<3, true>(a, v, n_items, quads, s) : launch_vt<3, false>(a, v, n_items, quads, s);
    case 4: return aff ? launch_vt<4, true>(a, v, n_items, quads, s) : launch_vt<4, false>(a, v, n_items, quads, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace wushkv
