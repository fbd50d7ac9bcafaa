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
// Work items: a unit's cache is a sequence of items -- packed blocks of 64
// tokens and window chunks of 8 fp16 tokens, each about 4 KB -- with the
// window chunks spread evenly among the packed blocks.  The units' items are
// laid end to end and CTA i of the one-wave grid (one CTA per SM) takes the
// i-th equal share (stream-K): usually the end of one unit and the start of
// the next.  The CTA's share is cut into equal warp ranges; a range that
// crosses a unit boundary leaves the finished unit's state in a shared-memory
// boundary slot.  A warp streams its items through a ring of
// shared-memory stages filled by bulk asynchronous copies (the TMA engine)
// and runs them on tensor cores with mma.sync: packed blocks on the integer
// pipe (codes u8 x two int8 terms of the query for the scores; codes u8 x
// two u8 terms of p * scale for PV), window chunks on the fp16 pipe (rows
// exact, query and p as fp16 hi/lo pairs).  Both kinds update the same
// online-softmax state.  Each CTA merges its warps per unit segment and
// writes one (m, l, o) partial; the last CTA of a unit to finish merges that
// unit's partials (an arrival counter; no CTA ever waits on another).
#include "async_copy.cuh"
#include "decode_frag.cuh"

namespace wushkv {

namespace {

// Warps per CTA (one CTA per SM): as many two-stage copy rings as shared
// memory holds for the code width.
template <int BITS> struct Warps { static constexpr int N = BITS == 2 ? 16 : BITS == 3 ? 12 : 9; };
constexpr int UMAX = 4;          // unit segments prepared per batch
constexpr int PB = 64;           // packed tokens per block
constexpr int WC = WIN_BOX_ROWS; // window tokens per chunk
// A window chunk in a stage: K then V, each two 1 KB tiles (dims 0-63 and
// 64-127) of WC rows x 128 bytes in the 128-byte swizzle (16-byte chunk j of
// row i at chunk j ^ i), as the tensor-map copies write them.
constexpr int WIN_V = 2048;      // offset of the V tiles of a window chunk
constexpr int PS_LD = PB + 16;   // bytes per row of the per-warp P tile
constexpr int NSTAGE = 2;        // per-warp copy stages
// Copies a warp issues before its first item; the rest of its ring fills
// once the first copy has landed (at G = 8 that start measured faster, and
// its code allocates registers without spills).
template <int G> struct FirstCopies { static constexpr int N = G == 8 ? 1 : NSTAGE; };
constexpr uint32_t WAIT_POLLS = 1u << 22;
constexpr unsigned FULL_MASK = 0xffffffffu;
constexpr int PART = PARTIAL_FLOATS;  // floats per partial record (16-byte rows)

// One packed block in a stage, byte for byte the cache's block record: K
// planes, V planes, K meta, V meta (MB bytes per token).
template <int BITS, bool AFFINE = false>
struct StageLayout {
  static constexpr int W0 = BITS == 4 ? 4 : 2;           // width of plane 0
  static constexpr int LO = PB * 16 * W0;                 // plane-0 bytes (K or V)
  static constexpr int HI = BITS == 3 ? PB * 16 : 0;      // plane-1 bytes
  static constexpr int MB = AFFINE ? 4 : 2;
  static constexpr int K_LO = 0, K_HI = LO, V_LO = LO + HI, V_HI = 2 * LO + HI;
  static constexpr int K_META = 2 * (LO + HI), V_META = K_META + PB * MB;
  static constexpr int PACKED = V_META + PB * MB;
};
// Stage size: the larger packed record or a window chunk, in whole 1 KB
// swizzle atoms (stages start on 1 KB boundaries).
template <int BITS>
struct StageBytes {
  static constexpr int RAW = StageLayout<BITS, true>::PACKED > 2 * WIN_V ? StageLayout<BITS, true>::PACKED
                                                                         : 2 * WIN_V;
  static constexpr int BYTES = (RAW + 1023) / 1024 * 1024;
};

// Items of one unit segment of a CTA's batch: its first global item, item
// count and window split (the same for every unit when all sequences hold
// the same number of tokens).
struct SegGeom {
  uint32_t start;
  int ni, win_chunks, n_sink, n_win, n_packed, ring_first;
};

template <int BITS, int G>
struct Smem {
  static constexpr int NW = Warps<BITS>::N;
  SegGeom geom[UMAX];
  static constexpr int NT = (G + 3) / 4;   // n-tiles of 8 columns (4 heads x 2 terms)
  alignas(1024) unsigned char stage[NW][NSTAGE][StageBytes<BITS>::BYTES];
  int8_t qterm[UMAX][NT * 4][2][D];        // two int8 terms per head (padded heads = 0)
  __half qh[UMAX][NT * 4][2][D + 8];       // fp16 hi/lo terms per head (rows padded: banks)
  float qscale[UMAX][NT * 4];              // sigma / 254 per head
  float qsum[UMAX][NT * 4];                // sum of the quantised q per head
  uint8_t ps[NW][NT * 8][PS_LD];           // per-warp P terms [col][token]
  float sm[NW][G], sl[NW][G];              // per-warp softmax max / sum
  // a warp whose item range crosses the end of segment j leaves its partial
  // for segment j here (at most one warp per boundary)
  float bo[UMAX - 1][G][D];
  float bm[UMAX - 1][G], bl[UMAX - 1][G];
  int bused[UMAX - 1];
  int wseg[NW];                            // segment of each warp's final state (-1: none)
  alignas(8) uint64_t bar[NW][NSTAGE];
  uint64_t never;                          // a barrier nothing arrives on (fault injection)
  int is_last[UMAX];
  // CTA merge: weight of each warp's slot in each segment (0 for warps of
  // other segments) and of the boundary slots; each segment's maximum (an
  // ordered integer while the warps raise it) and sum
  float wf[UMAX][NW][G], bf[UMAX - 1][G];
  int segMi[UMAX][G];
  float segL[UMAX][G];
  // other CTAs holding items of each segment's unit (0: no exchange)
  int others[UMAX];
};

// A warp's final partial output goes into its own copy stages once its ring
// has drained (no other warp touches them); the CTA's merged numerator of
// segment j follows the slot in warp j's stages.
template <int BITS, int G>
__device__ __forceinline__ float (*warp_slot(Smem<BITS, G>& sh, int w))[D] {
  static_assert(2 * sizeof(float) * G * D <= sizeof(sh.stage[0]), "stage area too small");
  static_assert(UMAX <= Smem<BITS, G>::NW, "segments per batch");
  return reinterpret_cast<float(*)[D]>(&sh.stage[w][0][0]);
}
template <int BITS, int G>
__device__ __forceinline__ float (*segment_sum(Smem<BITS, G>& sh, int j))[D] {
  return warp_slot(sh, j) + G;
}

// Order-preserving map of floats to ints (for integer max); -inf maps below
// every finite value.
__device__ __forceinline__ int float_order(float x) {
  const int i = __float_as_int(x);
  return i >= 0 ? i : i ^ 0x7FFFFFFF;
}
__device__ __forceinline__ float order_float(int i) { return __int_as_float(i >= 0 ? i : i ^ 0x7FFFFFFF); }

// Raise segment j's maximum to the warp's reference maxima (lanes 0..3
// hold head 4 nt + lane).
template <int BITS, int G>
__device__ __forceinline__ void raise_segment_max(Smem<BITS, G>& sh, int j, const float* m, int lane) {
  constexpr int NT = (G + 3) / 4;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
    if (lane < 4 && nt * 4 + lane < G) atomicMax(&sh.segMi[j][nt * 4 + lane], float_order(m[nt]));
}



// 2^x with the SFU (approximate, flushes denormal results to zero; 2^-inf = 0).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// Online-softmax state of a warp.  m is a reference maximum raised lazily:
// only when a score exceeds it by more than TAU (log2 units), so weights
// p = 2^(s - m) stay below 2^TAU and most items need no rescale.  In KEEP
// mode the packed blocks' PV products stay in int32 accumulators across
// items, all at the P scale F (a power of two bounding every p * scale
// quantised since the last flush); they are converted and added into o only
// when F or m changes, every FLUSH_BLOCKS blocks, and at the end.  Otherwise
// each block is quantised at its own maximum F and flushed at once.
constexpr float TAU = 8.f;
constexpr int FLUSH_BLOCKS = 256;  // int32 headroom: 256 blocks x 64 tokens x 255 x 240 < 2^31

template <int NT>
struct SoftmaxState {
  float m[NT], l[NT], e[NT], o[NT][8][2];   // o: dims 16mt + r (+8) of head 4nt + c
  float F[NT];                              // P scale of the pending int32 products (0: none)
  int pacc[8][NT][4];                       // pending PV products (KEEP only)
  int nacc;                                 // packed blocks since the last flush
};

// Smallest power of two >= x (x > 0, finite).
__device__ __forceinline__ float pow2_ceil(float x) {
  return __int_as_float((__float_as_int(x) + 0x007FFFFF) & 0x7F800000);
}

// Add the pending int32 PV products of n-tile nt (two byte terms, units of
// F / 65535) into o and clear them.
template <int NT>
__device__ __forceinline__ void flush_pv(SoftmaxState<NT>& S, int nt) {
  const float f = S.F[nt] * (1.f / 65535.f);
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    S.o[nt][mt][0] = fmaf(f, fmaf((float)S.pacc[mt][nt][0], 256.f, (float)S.pacc[mt][nt][1]), S.o[nt][mt][0]);
    S.o[nt][mt][1] = fmaf(f, fmaf((float)S.pacc[mt][nt][2], 256.f, (float)S.pacc[mt][nt][3]), S.o[nt][mt][1]);
    S.pacc[mt][nt][0] = S.pacc[mt][nt][1] = S.pacc[mt][nt][2] = S.pacc[mt][nt][3] = 0;
  }
}

// Raise the reference maximum of every n-tile to at least its score maximum
// over the warp (lm: this lane's), rescaling what was accumulated under the
// old one.  Called only when some lane's score exceeds m + TAU.
template <int NT, bool KEEP>
__device__ __forceinline__ void raise_max(SoftmaxState<NT>& S, const float (&lm)[NT]) {
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float bm = lm[nt];
    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 4));
    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 8));
    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 16));
    const float mn = fmaxf(S.m[nt], bm);
    if constexpr (KEEP) {
      if (S.F[nt] > 0.f) flush_pv(S, nt);
      S.F[nt] = 0.f;
    }
    const float al = S.m[nt] == mn ? 1.f : ex2(S.m[nt] - mn);   // 0 while m is still -inf
    S.l[nt] *= al;
    S.e[nt] *= al;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) { S.o[nt][mt][0] *= al; S.o[nt][mt][1] *= al; }
    S.m[nt] = mn;
  }
}

// As raise_max, for scores held as differences d = s - m_used from the
// reference in use (m_used = m, or 0 while m is still -inf): raises m to
// the warp's score maximum when that is higher and shifts the lane's
// differences dv to the new reference.
template <int NT, bool KEEP, int NV>
__device__ __forceinline__ void raise_max_d(SoftmaxState<NT>& S, const float (&lm)[NT],
                                            float (&dv)[NV][NT]) {
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float bm = lm[nt];
    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 4));
    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 8));
    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 16));
    const float mu = S.m[nt] == -INFINITY ? 0.f : S.m[nt];
    const float mn = fmaxf(S.m[nt], mu + bm);
    if (mn == S.m[nt]) continue;
    if constexpr (KEEP) {
      if (S.F[nt] > 0.f) flush_pv(S, nt);
      S.F[nt] = 0.f;
    }
    const float al = ex2(S.m[nt] - mn);   // 0 while m is still -inf
    S.l[nt] *= al;
    S.e[nt] *= al;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) { S.o[nt][mt][0] *= al; S.o[nt][mt][1] *= al; }
    S.m[nt] = mn;
    if (mn != -INFINITY) {
      const float sh = mn - mu;
#pragma unroll
      for (int v = 0; v < NV; ++v) dv[v][nt] -= sh;
    }
  }
}

__device__ __forceinline__ float merge_weight(float m, float M) {
  return (m == -INFINITY) ? 0.f : ex2(m - M);
}

// Stream-K split of the items laid end to end: the first cta_r CTAs take
// cta_q + 1 items, the others cta_q (cta_q >= 1).  All indices fit in 32
// bits (the host refuses larger problems).
__device__ __forceinline__ uint32_t cta_begin(const DecodeArgs& a, uint32_t cta) {
  return cta * a.cta_q + min(cta, a.cta_r);
}
// CTA whose item range contains global item y.
__device__ __forceinline__ uint32_t cta_of(const DecodeArgs& a, uint32_t y) {
  const uint32_t big = a.cta_r * (a.cta_q + 1);
  return y < big ? y / (a.cta_q + 1) : a.cta_r + (y - big) / a.cta_q;
}

// Item i of a unit (0 <= i < ni = win_chunks + pack_blocks) is window chunk
// number W(i) = floor(i nw / ni) when W steps up at i, else packed block
// i - W(i).  A cursor walks a warp's items in order, keeping W(i) as a
// quotient and remainder: one division when it starts, then an add and a
// compare per item.
struct ItemCursor {
  int i, w, rem;   // current item, W(i), i nw - W(i) ni
  template <bool MAYBE_EMPTY = true>   // false: ni > 0 is known
  __device__ __forceinline__ void start(int ni_, int win_chunks, int i0) {
    const uint32_t ni = ni_;
    const uint32_t x = (uint32_t)i0 * (uint32_t)win_chunks;   // < 2^32 (host check)
    i = i0;
    w = (!MAYBE_EMPTY || ni) ? (int)(x / ni) : 0;
    rem = (int)(x - (uint32_t)w * ni);
  }
  // Classify the current item (window chunk or packed block, and its
  // number), then step to the next.
  __device__ __forceinline__ bool take(int ni, int win_chunks, int* idx) {
    rem += win_chunks;
    const bool win = rem >= ni;
    *idx = win ? w : i - w;
    if (win) { rem -= ni; ++w; }
    ++i;
    return win;
  }
};

__device__ __forceinline__ const __half* window_row(const DevCache& c, int n_sink, int ring_first,
                                                    const __half* sink, const __half* ring, int u, int w) {
  if (w < n_sink) return sink + ((size_t)u * c.sink + w) * D;
  int slot = ring_first + (w - n_sink);   // < 2 ring_slots
  if (slot >= c.ring_slots) slot -= c.ring_slots;
  return ring + ((size_t)u * c.ring_slots + slot) * D;
}

// All lanes: copy an item of unit u (window chunk or packed block number idx)
// into a stage.  A packed block is one bulk copy of its block record.  A
// window chunk whose valid rows are consecutive in the sink or the ring
// (the usual case) is four tensor-map copies; any other chunk (it straddles
// the sink and the ring, or the ring's wrap) is gathered by the warp with
// plain loads into the same swizzled tiles.  Rows past the window are
// whatever the box covers there (zeros outside the array, else stale but
// finite rows, the buffer being zeroed at creation) or, when gathered, the
// window's last row; their scores are masked.
template <int BITS, bool AFFINE, class GEO>
__device__ __forceinline__ void issue_item(const DecodeArgs& a, const GEO& geo, int j, const WindowMaps& wm,
                                           bool win, int idx, unsigned char* st, uint64_t* bar, int lane) {
  using SL = StageLayout<BITS, AFFINE>;
  const DevCache& c = a.c;
  const int u = geo.u_first + j;
  if (win) {
    const int nwin = geo.n_win(j), n_sink = geo.n_sink(j);
    const int w0 = idx * WC, w1 = min(w0 + WC, nwin) - 1;
    const CUtensorMap* mk = nullptr;
    const CUtensorMap* mv = nullptr;
    int y = 0;
    if (w1 < n_sink) {
      if (wm.has_sink) { mk = &wm.sink_k; mv = &wm.sink_v; y = u * c.sink + w0; }
    } else if (w0 >= n_sink) {
      int s0 = geo.ring_first(j) + (w0 - n_sink);
      if (s0 >= c.ring_slots) s0 -= c.ring_slots;
      if (wm.has_ring && s0 + (w1 - w0) < c.ring_slots) {
        mk = &wm.ring_k; mv = &wm.ring_v; y = u * c.ring_slots + s0;
      }
    }
    if (mk != nullptr) {
      if (lane == 0) {
        const uint64_t pol = l2_evict_first_policy();
        mbar_arrive_expect_tx(bar, 2u * WIN_V);
        tma_load_2d_hint(st, mk, 0, y, bar, pol);
        tma_load_2d_hint(st + 1024, mk, 64, y, bar, pol);
        tma_load_2d_hint(st + WIN_V, mv, 0, y, bar, pol);
        tma_load_2d_hint(st + WIN_V + 1024, mv, 64, y, bar, pol);
      }
      return;
    }
    for (int e = lane; e < 2 * WC * 16; e += 32) {
      const int kv = e / (WC * 16), j = (e / 16) % WC, q = e % 16;
      const int w = min(w0 + j, nwin - 1);
      const __half* row = window_row(c, n_sink, geo.ring_first(j), kv ? c.sink_v : c.sink_k,
                                     kv ? c.ring_v : c.ring_k, u, w);
      const uint4 val = *reinterpret_cast<const uint4*>(row + 8 * q);
      *reinterpret_cast<uint4*>(st + kv * WIN_V + (q / 8) * 1024 + j * 128 + (((q % 8) ^ j) * 16)) = val;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive_once(bar);
    return;
  }
  if (lane != 0) return;
  mbar_arrive_expect_tx(bar, (uint32_t)SL::PACKED);
  // (the general variant may read a paged region; the uniform one is dense)
  const uint64_t off = GEO::kTable ? block_offset(c, u, idx)
                                   : (uint64_t)u * c.unit_stride + (uint64_t)idx * c.block_stride;
  bulk_copy_g2s_hint(st, c.k_plane[0] + off, (uint32_t)SL::PACKED, bar, l2_evict_first_policy());
}

// ---- packed blocks: copy ring + integer tensor cores ------------------------------
// K row words of token row t for lane c4 (3- and 4-bit keys; 2-bit keys are
// read as quads in packed_block_compute).
template <int BITS>
__device__ __forceinline__ KWords<BITS> stage_k_words(const unsigned char* st, int t, int c4) {
  static_assert(BITS == 3 || BITS == 4, "2-bit keys are packed in quads");
  using SL = StageLayout<BITS>;
  KWords<BITS> w;
  if constexpr (BITS == 3) {
    w.lo = *reinterpret_cast<const uint2*>(st + SL::K_LO + t * 32 + 8 * c4);
    w.hi = *reinterpret_cast<const uint32_t*>(st + SL::K_HI + t * 16 + 4 * c4);
  } else {
    w.w = *reinterpret_cast<const uint4*>(st + SL::K_LO + t * 64 + 16 * c4);
  }
  return w;
}

// V quad qi (0..15) of the block, row unit of lane row r at rotated position pos.
template <int BITS>
__device__ __forceinline__ VWords<BITS> stage_v_words(const unsigned char* st, int qi, int pos) {
  using SL = StageLayout<BITS>;
  VWords<BITS> v;
  if constexpr (BITS == 2) {
    v.lo = *reinterpret_cast<const uint4*>(st + SL::V_LO + qi * 128 + pos * 16);
  } else if constexpr (BITS == 3) {
    v.lo = *reinterpret_cast<const uint4*>(st + SL::V_LO + qi * 128 + pos * 16);
    v.hi = *reinterpret_cast<const uint2*>(st + SL::V_HI + qi * 64 + pos * 8);
  } else {
    v.a = *reinterpret_cast<const uint4*>(st + SL::V_LO + qi * 256 + pos * 16);
    v.b = *reinterpret_cast<const uint4*>(st + SL::V_LO + qi * 256 + 128 + pos * 16);
  }
  return v;
}


// Token (within the block) of slot j = 2 mt + th of lane row r: 2-bit keys
// come in quads (m-tile mt = field mt of quads r and r + 8), wider keys in
// rows (8 consecutive tokens per lane).
template <int BITS>
__device__ __forceinline__ int slot_token(int r, int j) {
  if constexpr (BITS == 2) return 4 * r + 32 * (j & 1) + (j >> 1);
  else return 8 * r + j;
}

// Lane = 4r + c.  Score m-tile rows r, r+8 are tokens; columns are (head,
// term) pairs, so thread c owns head 4nt + c of n-tile nt.  PV m-tile rows
// are dims 16mt + r (+8); the PV B operand comes back through the warp's P
// tile in shared memory.  FULL: all 64 tokens of the block are cached.
template <int BITS, int G, bool AFFINE, bool FULL, bool KEEP>
__device__ __forceinline__ void packed_block_compute(
    const DecodeArgs& a, Smem<BITS, G>& sh, const unsigned char* st, int blk, int warp, int lane,
    const uint32_t (&qb)[(G + 3) / 4][4][2], const float (&qscale)[(G + 3) / 4],
    const float (&qoff)[(G + 3) / 4], const float (&qsum)[(G + 3) / 4], SoftmaxState<(G + 3) / 4>& S,
    int n_packed) {
  constexpr int NT = (G + 3) / 4;
  using SL = StageLayout<BITS, AFFINE>;
  const int r = lane >> 2, c4 = lane & 3;
  const int nvalid = n_packed - blk * PB;  // used when !FULL

  // ---- scores ----------------------------------------------------------------
  // Lane 4r + c owns eight tokens of the block: slot j = 2 mt + th is row
  // r + 8 th of m-tile mt, token slot_token(r, j).  2-bit keys: the lane
  // reads its eight words of quads r and r + 8 as four 16-byte chunks.
  // Wider keys: its K rows sit at positions 8r + (j ^ (r & 3)) (the cache's
  // row swizzle), which spreads each load over all shared-memory banks.
  // sc[j]: score minus the reference in use (m, or 0 while m = -inf)
  float sc[8][NT];
  float vs[8], vo[8];
  float nm[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) nm[nt] = S.m[nt] == -INFINITY ? 0.f : -S.m[nt];
  {   // per-token meta of the lane's eight tokens: two 16-byte loads (QuEST)
    float ks_[8], ko_[8];
    if constexpr (AFFINE) {
#pragma unroll
      for (int hq = 0; hq < 2; ++hq) {   // four consecutive tokens per load (slot_token)
        const int off = BITS == 2 ? 16 * r + 128 * hq : 32 * r + 16 * hq;
        const uint4 km = *reinterpret_cast<const uint4*>(st + SL::K_META + off);
        const uint4 vm = *reinterpret_cast<const uint4*>(st + SL::V_META + off);
        const uint32_t kw[4] = {km.x, km.y, km.z, km.w}, vw[4] = {vm.x, vm.y, vm.z, vm.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = BITS == 2 ? 2 * e + hq : 4 * hq + e;
          const float2 kf = __half22float2(*reinterpret_cast<const __half2*>(&kw[e]));
          const float2 vf = __half22float2(*reinterpret_cast<const __half2*>(&vw[e]));
          ks_[j] = kf.x; ko_[j] = kf.y;
          vs[j] = vf.x; vo[j] = vf.y;
        }
      }
    } else if constexpr (BITS == 2) {
      // the lane's tokens 4r .. 4r + 3 (th = 0) and 4r + 32 .. 4r + 35 (th = 1)
#pragma unroll
      for (int th = 0; th < 2; ++th) {
        const uint2 km = *reinterpret_cast<const uint2*>(st + SL::K_META + 8 * r + 64 * th);
        const uint2 vm = *reinterpret_cast<const uint2*>(st + SL::V_META + 8 * r + 64 * th);
        const float2 k01 = __half22float2(*reinterpret_cast<const __half2*>(&km.x));
        const float2 k23 = __half22float2(*reinterpret_cast<const __half2*>(&km.y));
        const float2 v01 = __half22float2(*reinterpret_cast<const __half2*>(&vm.x));
        const float2 v23 = __half22float2(*reinterpret_cast<const __half2*>(&vm.y));
        ks_[th] = k01.x; ks_[2 + th] = k01.y; ks_[4 + th] = k23.x; ks_[6 + th] = k23.y;
        vs[th] = v01.x; vs[2 + th] = v01.y; vs[4 + th] = v23.x; vs[6 + th] = v23.y;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) ko_[j] = vo[j] = 0.f;
    } else {
      const uint4 km = *reinterpret_cast<const uint4*>(st + SL::K_META + 16 * r);
      const uint4 vm = *reinterpret_cast<const uint4*>(st + SL::V_META + 16 * r);
      const uint32_t kw[4] = {km.x, km.y, km.z, km.w}, vw[4] = {vm.x, vm.y, vm.z, vm.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 kf = __half22float2(*reinterpret_cast<const __half2*>(&kw[e]));
        const float2 vf = __half22float2(*reinterpret_cast<const __half2*>(&vw[e]));
        ks_[2 * e] = kf.x; ks_[2 * e + 1] = kf.y;
        vs[2 * e] = vf.x; vs[2 * e + 1] = vf.y;
        ko_[2 * e] = ko_[2 * e + 1] = vo[2 * e] = vo[2 * e + 1] = 0.f;
      }
    }
    // K fragments of m-tile mt, k-step ks: rows r, r + 8 are tokens
    // slot_token(r, 2 mt), slot_token(r, 2 mt + 1); 2-bit words carry the
    // m-tile's field in place (times 4^mt, removed with the query scale)
    uint32_t wr[4][2], w8[4][2];   // 2-bit: words [ks][h] of quads r and r + 8
    if constexpr (BITS == 2) {
      const int xq = r & 1;
      const unsigned char* q0 = st + SL::K_LO + r * 128;
      const unsigned char* q1 = st + SL::K_LO + (r + 8) * 128;
      const uint4 a0 = *reinterpret_cast<const uint4*>(q0 + ((2 * c4) ^ xq) * 16);
      const uint4 a1 = *reinterpret_cast<const uint4*>(q0 + ((2 * c4 + 1) ^ xq) * 16);
      const uint4 b0 = *reinterpret_cast<const uint4*>(q1 + ((2 * c4) ^ xq) * 16);
      const uint4 b1 = *reinterpret_cast<const uint4*>(q1 + ((2 * c4 + 1) ^ xq) * 16);
      wr[0][0] = a0.x; wr[0][1] = a0.y; wr[1][0] = a0.z; wr[1][1] = a0.w;
      wr[2][0] = a1.x; wr[2][1] = a1.y; wr[3][0] = a1.z; wr[3][1] = a1.w;
      w8[0][0] = b0.x; w8[0][1] = b0.y; w8[1][0] = b0.z; w8[1][1] = b0.w;
      w8[2][0] = b1.x; w8[2][1] = b1.y; w8[3][0] = b1.z; w8[3][1] = b1.w;
    }
    const int x = r & 3;
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      int acc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0;
      if constexpr (BITS == 2) {
        const uint32_t m = 0x03030303u << (2 * mt);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint32_t a0 = wr[ks][0] & m, a1 = w8[ks][0] & m, a2 = wr[ks][1] & m, a3 = w8[ks][1] & m;
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) mma_u8s8(acc[nt], a0, a1, a2, a3, qb[nt][ks][0], qb[nt][ks][1]);
        }
      } else {
        const KWords<BITS> kw0 = stage_k_words<BITS>(st, 8 * r + ((2 * mt) ^ x), c4);
        const KWords<BITS> kw1 = stage_k_words<BITS>(st, 8 * r + ((2 * mt + 1) ^ x), c4);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint32_t a0 = k_frag<BITS>(kw0, ks, 0), a1 = k_frag<BITS>(kw1, ks, 0);
          const uint32_t a2 = k_frag<BITS>(kw0, ks, 1), a3 = k_frag<BITS>(kw1, ks, 1);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) mma_u8s8(acc[nt], a0, a1, a2, a3, qb[nt][ks][0], qb[nt][ks][1]);
        }
      }
      constexpr float kf4[4] = {1.f, 0.25f, 0.0625f, 0.015625f};
      const float fmt = BITS == 2 ? kf4[mt] : 1.f;   // 4^-mt (exact)
#pragma unroll
      for (int th = 0; th < 2; ++th) {
        const int j = 2 * mt + th;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const float xf = (float)(acc[nt][2 * th] * 254 + acc[nt][2 * th + 1]);
          const float qsc = qscale[nt] * fmt;
          float d;   // score minus the reference maximum in use
          if constexpr (AFFINE) d = fmaf(ks_[j], qsc * xf, fmaf(ko_[j], qsum[nt], nm[nt]));
          else d = fmaf(ks_[j], fmaf(qsc, xf, qoff[nt]), nm[nt]);   // delta (q.c + beta sum q) - m
          if constexpr (!FULL) d = (slot_token<BITS>(r, j) < nvalid) ? d : -INFINITY;
          sc[j][nt] = d;
        }
      }
    }
  }

  // ---- online softmax; P as 16-bit fixed point in two byte terms ---------------
  // Votes keep the common item free of cross-lane reductions: the maximum
  // is reduced only when some score passes m + TAU, the P scale only when
  // some p * scale passes F.
  {
    float lm[NT];
    bool up = false;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float x = -INFINITY;
#pragma unroll
      for (int v = 0; v < 8; ++v) x = fmaxf(x, sc[v][nt]);
      lm[nt] = x;
      up |= x > TAU || S.m[nt] == -INFINITY;
    }
    if (__any_sync(FULL_MASK, up)) raise_max_d<NT, KEEP, 8>(S, lm, sc);
  }
  uint8_t* ps = &sh.ps[warp][0][0];
  float pmx[NT];
  bool grow = false;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float ls = 0.f, es = 0.f, pm = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float p = ex2(sc[j][nt]);   // masked tokens: exp2(-inf) = 0
      float pt = p * vs[j];
      if constexpr (!FULL) pt = (slot_token<BITS>(r, j) < nvalid) ? pt : 0.f;
      ls += p;
      if constexpr (AFFINE) es = fmaf(p, vo[j], es);
      else es += pt;                                 // times beta at the end
      pm = fmaxf(pm, pt);
      sc[j][nt] = pt;
    }
    S.l[nt] += ls;
    S.e[nt] += es;
    pmx[nt] = pm;
    grow |= pm > S.F[nt];
  }
  if (KEEP ? __any_sync(FULL_MASK, grow) : true) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float pm = pmx[nt];
      pm = fmaxf(pm, __shfl_xor_sync(FULL_MASK, pm, 4));
      pm = fmaxf(pm, __shfl_xor_sync(FULL_MASK, pm, 8));
      pm = fmaxf(pm, __shfl_xor_sync(FULL_MASK, pm, 16));
      if constexpr (KEEP) {
        if (pm > S.F[nt]) {
          if (S.F[nt] > 0.f) flush_pv(S, nt);
          S.F[nt] = pow2_ceil(pm);
        }
      } else {
        S.F[nt] = pm;
      }
    }
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    // 65535 / F: exact for the power-of-two F of KEEP mode; otherwise the
    // correctly rounded reciprocal keeps pt * inv <= 65535 (1 + 2^-23)
    float inv = 0.f;
    if (S.F[nt] > 0.f)
      inv = KEEP ? 65535.f * __int_as_float(0x7F000000 - __float_as_int(S.F[nt])) : 65535.f * __frcp_rn(S.F[nt]);
    // 1.5 * 2^23 + rint(pt * 65535 / F): the low 16 mantissa bits are the
    // rounded value; its high byte is term 0, its low byte term 1.  Bytes of
    // four tokens are gathered into one word per term.
    uint32_t bw[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) bw[j] = __float_as_uint(fmaf(sc[j][nt], inv, 12582912.f));
    uint32_t t0w[2], t1w[2];
#pragma unroll
    for (int hq = 0; hq < 2; ++hq) {   // four consecutive tokens (slot_token) per word
      const int j0 = BITS == 2 ? hq : 4 * hq, dj = BITS == 2 ? 2 : 1;
      const uint32_t x01 = __byte_perm(bw[j0], bw[j0 + dj], 0x5140);               // lo0 lo1 hi0 hi1
      const uint32_t x23 = __byte_perm(bw[j0 + 2 * dj], bw[j0 + 3 * dj], 0x5140);  // lo2 lo3 hi2 hi3
      t1w[hq] = __byte_perm(x01, x23, 0x5410);
      t0w[hq] = __byte_perm(x01, x23, 0x7632);
    }
    const int col = nt * 8 + 2 * c4;
    if constexpr (BITS == 2) {   // tokens 4r .. 4r + 3 and 4r + 32 .. 4r + 35
      *reinterpret_cast<uint32_t*>(ps + col * PS_LD + 4 * r) = t0w[0];
      *reinterpret_cast<uint32_t*>(ps + col * PS_LD + 4 * r + 32) = t0w[1];
      *reinterpret_cast<uint32_t*>(ps + (col + 1) * PS_LD + 4 * r) = t1w[0];
      *reinterpret_cast<uint32_t*>(ps + (col + 1) * PS_LD + 4 * r + 32) = t1w[1];
    } else {
      *reinterpret_cast<uint2*>(ps + col * PS_LD + 8 * r) = make_uint2(t0w[0], t0w[1]);
      *reinterpret_cast<uint2*>(ps + (col + 1) * PS_LD + 8 * r) = make_uint2(t1w[0], t1w[1]);
    }
  }
  __syncwarp();

  // ---- PV: dims x (head, term) over the 64 tokens ------------------------------
  if constexpr (!KEEP) {
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        S.pacc[mt][nt][0] = S.pacc[mt][nt][1] = S.pacc[mt][nt][2] = S.pacc[mt][nt][3] = 0;
  }
  const int pos = (r + 2 * c4) & 7;  // rotated row unit (quads 8k2 + c4 + 4q all have quad & 3 == c4)
#pragma unroll
  for (int k2 = 0; k2 < 2; ++k2) {
    const VWords<BITS> v0 = stage_v_words<BITS>(st, 8 * k2 + c4, pos);
    const VWords<BITS> v1 = stage_v_words<BITS>(st, 8 * k2 + c4 + 4, pos);
    uint32_t pb[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const uint8_t* row = ps + (nt * 8 + r) * PS_LD + 32 * k2 + 4 * c4;
      pb[nt][0] = *reinterpret_cast<const uint32_t*>(row);
      pb[nt][1] = *reinterpret_cast<const uint32_t*>(row + 16);
    }
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      uint32_t a0, a1, a2, a3;
      if constexpr (BITS == 3) {
        a0 = v_frag<BITS>(v0, 2 * mt); a1 = v_frag<BITS>(v0, 2 * mt + 1);
        a2 = v_frag<BITS>(v1, 2 * mt); a3 = v_frag<BITS>(v1, 2 * mt + 1);
      } else {
        a0 = v_frag_scaled<BITS>(v0, 2 * mt); a1 = v_frag_scaled<BITS>(v0, 2 * mt + 1);
        a2 = v_frag_scaled<BITS>(v1, 2 * mt); a3 = v_frag_scaled<BITS>(v1, 2 * mt + 1);
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_u8u8(S.pacc[mt][nt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
    }
  }
  __syncwarp();
  if constexpr (KEEP) {
    if (++S.nacc == FLUSH_BLOCKS) {
      S.nacc = 0;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) flush_pv(S, nt);
    }
  } else {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) flush_pv(S, nt);
  }
}

// Power-of-two factor of a PV dim row in the packed path (shift-free
// fragments); window contributions are brought to the same units.
template <int BITS>
__device__ __forceinline__ float row_factor(int rho) {
  if constexpr (BITS == 3) return 1.f;
  else return 1.f / v_row_scale<BITS>(rho);
}

// One window chunk (8 fp16 tokens) from its stage: scores with fp16 MMA
// (rows 8-15 of the m16 tile are empty), PV with the transposed rows.
template <int BITS, int G, bool KEEP>
__device__ __forceinline__ void window_chunk_compute(const DecodeArgs& a, Smem<BITS, G>& sh,
                                                     const unsigned char* st, int wc, int j, int lane,
                                                     SoftmaxState<(G + 3) / 4>& S, int n_win) {
  constexpr int NT = (G + 3) / 4;
  const int r = lane >> 2, c4 = lane & 3;
  const bool valid = wc * WC + r < n_win;
  // lane supplies row j = lane % 8 of matrix lane / 8 (dims 32kk + 8 (lane / 8)
  // .. +7: 16-byte chunk 4 (kk % 2) + lane / 8 of tile kk / 2, swizzled with j;
  // odd kk flips bit 2 of the chunk, i.e. bit 6 of the 1 KB-aligned address)
  const int j8 = lane & 7;
  const uint32_t row_addr = smem_addr(st) + j8 * 128 + (((lane >> 3) ^ j8) << 4);

  float acc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    uint32_t kf[4];
    ldmatrix_x4(kf, (row_addr ^ ((kk & 1) << 6)) + (kk >> 1) * 1024);   // dims 32kk .. 32kk + 31
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int ks = 2 * kk + hf;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const __half* qrow = &sh.qh[j][nt * 4 + (r >> 1)][r & 1][16 * ks + 2 * c4];
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(qrow);
        const uint32_t b1 = *reinterpret_cast<const uint32_t*>(qrow + 8);
        mma_f16_k16(acc[nt], kf[2 * hf], 0u, kf[2 * hf + 1], 0u, b0, b1);
      }
    }
  }

  float sv[NT];
  {
    bool up = false;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      sv[nt] = valid ? acc[nt][0] + acc[nt][1] : -INFINITY;   // hi + lo query terms
      up |= sv[nt] > S.m[nt] + TAU;
    }
    if (__any_sync(FULL_MASK, up)) raise_max<NT, KEEP>(S, sv);
  }
  uint32_t pb[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const float p = valid ? ex2(sv[nt] - S.m[nt]) : 0.f;
    S.l[nt] += p;
    // B fragment of PV: p of tokens 2c, 2c+1 for column r = (head r/2, term r%2)
    const float pa = __shfl_sync(FULL_MASK, p, 8 * c4 + (r >> 1));
    const float pc = __shfl_sync(FULL_MASK, p, 8 * c4 + 4 + (r >> 1));
    __half ha = __float2half_rn(pa), hc = __float2half_rn(pc);
    if (r & 1) {
      ha = __float2half_rn(pa - __half2float(ha));
      hc = __float2half_rn(pc - __half2float(hc));
    }
    const __half2 h2 = __halves2half2(ha, hc);
    pb[nt] = *reinterpret_cast<const uint32_t*>(&h2);
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t vf[4];
    ldmatrix_x4_trans(vf, (row_addr ^ ((q & 1) << 6)) + WIN_V + (q >> 1) * 1024);   // dims 32q .. 32q + 31
#pragma unroll
    for (int hm = 0; hm < 2; ++hm) {
      const int mt = 2 * q + hm;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float d[4] = {0.f, 0.f, 0.f, 0.f};
        mma_f16_k8(d, vf[2 * hm], vf[2 * hm + 1], pb[nt]);
        S.o[nt][mt][0] = fmaf(row_factor<BITS>(2 * mt), d[0] + d[1], S.o[nt][mt][0]);
        S.o[nt][mt][1] = fmaf(row_factor<BITS>(2 * mt + 1), d[2] + d[3], S.o[nt][mt][1]);
      }
    }
  }
}

// Item geometry of the batch's unit segments: from the kernel arguments
// when every sequence holds the same number of tokens, else from the
// per-batch table in shared memory.
template <bool RAGGED, int BITS, int G>
struct Geo {
  static constexpr bool kTable = RAGGED;
  const Smem<BITS, G>& sh;
  const DecodeArgs& a;
  int u_first;
  // (uniform sequences read the kernel arguments at each use)
  __device__ __forceinline__ int ni(int j) const { return RAGGED ? sh.geom[j].ni : a.items_per_unit; }
  __device__ __forceinline__ int win_chunks(int j) const { return RAGGED ? sh.geom[j].win_chunks : a.win_chunks; }
  __device__ __forceinline__ int n_sink(int j) const { return RAGGED ? sh.geom[j].n_sink : a.n_sink; }
  __device__ __forceinline__ int n_win(int j) const { return RAGGED ? sh.geom[j].n_win : a.n_sink + a.n_recent; }
  __device__ __forceinline__ int n_packed(int j) const { return RAGGED ? sh.geom[j].n_packed : a.n_packed; }
  __device__ __forceinline__ int ring_first(int j) const { return RAGGED ? sh.geom[j].ring_first : a.ring_first; }
  __device__ __forceinline__ uint32_t start(int j) const {
    return RAGGED ? sh.geom[j].start : (uint32_t)(u_first + j) * (uint32_t)a.items_per_unit;
  }
  __device__ __forceinline__ SegGeom operator()(int j) const {
    SegGeom g;
    g.ni = ni(j); g.start = start(j); g.win_chunks = win_chunks(j); g.n_sink = n_sink(j);
    g.n_win = n_win(j); g.n_packed = n_packed(j); g.ring_first = ring_first(j);
    return g;
  }
  // segment holding global item y (segments without items are stepped over)
  __device__ __forceinline__ int segment_of(uint32_t y) const {
    if constexpr (RAGGED) {
      int j = 0;
      while (y >= sh.geom[j].start + (uint32_t)sh.geom[j].ni) ++j;
      return j;
    } else {
      return (int)(y / (uint32_t)a.items_per_unit) - u_first;
    }
  }
};

// Cursor over items laid end to end across the batch's unit segments.
struct GCursor {
  int j;
  ItemCursor ic;
  template <class GEO>
  __device__ __forceinline__ void start(const GEO& geo, uint32_t y) {
    j = geo.segment_of(y);
    ic.start<GEO::kTable>(geo.ni(j), geo.win_chunks(j), (int)(y - geo.start(j)));
  }
  template <class GEO>
  __device__ __forceinline__ bool take(const GEO& geo, int* idx, int* seg) {
    if constexpr (GEO::kTable) {   // a table may hold units without items
      while (ic.i == geo.ni(j)) { ++j; ic.start<true>(geo.ni(j), geo.win_chunks(j), 0); }
    } else {
      if (ic.i == geo.ni(j)) { ++j; ic.start<false>(geo.ni(j), geo.win_chunks(j), 0); }
    }
    *seg = j;
    return ic.take(geo.ni(j), geo.win_chunks(j), idx);
  }
};

// First copies of the warp's items [y0, y1), issued before the query prologue.
template <int BITS, bool AFFINE, int G, class GEO>
__device__ __forceinline__ void warp_items_prefetch(const DecodeArgs& a, const WindowMaps& wm,
                                                    Smem<BITS, G>& sh, const GEO& geo, uint32_t y0, uint32_t y1,
                                                    int warp, int lane, uint32_t it, GCursor& ic) {
  ic.start(geo, y0);
  for (uint32_t j = 0; j < (uint32_t)FirstCopies<G>::N && y0 + j < y1; ++j) {
    const int stg = (it + j) % NSTAGE;
    int idx, seg;
    const bool win = ic.take(geo, &idx, &seg);
    issue_item<BITS, AFFINE>(a, geo, seg, wm, win, idx, sh.stage[warp][stg], &sh.bar[warp][stg], lane);
  }
}

// Reset the softmax state and load the query registers of segment j.
template <int BITS, int G>
__device__ __forceinline__ void begin_segment(const Smem<BITS, G>& sh, int j, int lane,
                                              uint32_t (&qb)[(G + 3) / 4][4][2], float (&qscale)[(G + 3) / 4],
                                              float (&qsum)[(G + 3) / 4], float (&qoff)[(G + 3) / 4],
                                              SoftmaxState<(G + 3) / 4>& S) {
  constexpr int NT = (G + 3) / 4;
  const int r = lane >> 2, c4 = lane & 3;
  const float beta = 0.5f - (float)(1 << (BITS - 1));
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int gcol = nt * 4 + (r >> 1), term = r & 1;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
#pragma unroll
      for (int h = 0; h < 2; ++h)
        qb[nt][ks][h] = *reinterpret_cast<const uint32_t*>(&sh.qterm[j][gcol][term][32 * ks + 16 * h + 4 * c4]);
    qscale[nt] = sh.qscale[j][nt * 4 + c4];
    qsum[nt] = sh.qsum[j][nt * 4 + c4];
    qoff[nt] = beta * qsum[nt];
    S.m[nt] = -INFINITY; S.l[nt] = 0.f; S.e[nt] = 0.f; S.F[nt] = 0.f;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      S.o[nt][mt][0] = S.o[nt][mt][1] = 0.f;
      S.pacc[mt][nt][0] = S.pacc[mt][nt][1] = S.pacc[mt][nt][2] = S.pacc[mt][nt][3] = 0;
    }
  }
  S.nacc = 0;
}

// Write a warp's finished softmax state (all lanes) as one partial: o[g][d]
// (value-space numerator, offsets included), m[g], l[g].
template <int BITS, int G, bool AFFINE>
__device__ __forceinline__ void state_to_slot(const SoftmaxState<(G + 3) / 4>& S, float (*o)[D], float* m,
                                              float* l, int lane) {
  constexpr int NT = (G + 3) / 4;
  const int r = lane >> 2, c4 = lane & 3;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float lt = S.l[nt], et = S.e[nt];
#pragma unroll
    for (int sft = 4; sft < 32; sft <<= 1) {
      lt += __shfl_xor_sync(FULL_MASK, lt, sft);
      et += __shfl_xor_sync(FULL_MASK, et, sft);
    }
    if constexpr (!AFFINE) et *= 0.5f - (float)(1 << (BITS - 1));  // sum p*delta*beta
    const int g = nt * 4 + c4;
    if (g < G) {
      if (r == 0) { m[g] = S.m[nt]; l[g] = lt; }
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        o[g][16 * mt + r] = fmaf(S.o[nt][mt][0], 1.f / row_factor<BITS>(2 * mt), et);
        o[g][16 * mt + r + 8] = fmaf(S.o[nt][mt][1], 1.f / row_factor<BITS>(2 * mt + 1), et);
      }
    }
  }
}

// The warp's items [y0, y1) (global item indices, possibly spanning units)
// through its copy ring; the first NSTAGE copies were issued by
// warp_items_prefetch, whose cursor ic stands at the next item to copy.
// When the items move on to the next unit, the finished unit's state goes
// to that segment's boundary slot.  Returns the segment of the final state
// in S (-1 if the warp had no items).
template <int BITS, int G, bool AFFINE, class GEO>
__device__ int warp_run(const DecodeArgs& a, const WindowMaps& wm, Smem<BITS, G>& sh, const GEO& geo,
                        uint32_t y0, uint32_t y1, int warp, int lane, uint32_t& it, GCursor& ic,
                        SoftmaxState<(G + 3) / 4>& S) {
  constexpr int NT = (G + 3) / 4;
  // int32 PV accumulators kept across items: one n-tile (registers) and 2 or
  // 3 bits (with 4-bit codes the coarser shared P scale shows next to the
  // finer code grid, so those flush every block at its own exact scale)
  constexpr bool KEEP = NT == 1 && BITS <= 3;
  uint32_t qb[NT][4][2];
  float qscale[NT], qsum[NT], qoff[NT];
  if (y1 <= y0) return -1;
  int cur = -1;
  uint32_t y = y0;
  while (y < y1) {   // one piece per unit the range touches
    const int j = geo.segment_of(y);
    const uint32_t yend = min(y1, geo.start(j) + (uint32_t)geo.ni(j));
    if (cur >= 0) {   // leaving segment cur: its state goes to the boundary slot
      if constexpr (KEEP) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          if (S.F[nt] > 0.f) flush_pv(S, nt);
      }
      state_to_slot<BITS, G, AFFINE>(S, sh.bo[cur], sh.bm[cur], sh.bl[cur], lane);
      raise_segment_max(sh, cur, S.m, lane);
      if (lane == 0) sh.bused[cur] = 1;
    }
    begin_segment<BITS, G>(sh, j, lane, qb, qscale, qsum, qoff, S);
    cur = j;
    ItemCursor cc;
    cc.start<false>(geo.ni(j), geo.win_chunks(j), (int)(y - geo.start(j)));
    for (; y < yend; ++y, ++it) {
      const int stg = it % NSTAGE;
      // (fault injection for tests: the warp's first wait is made on a
      // barrier that nothing completes, so it runs out)
      const bool injected = a.inject_polls != 0 && y == y0;
      if (!mbar_wait_bounded(injected ? &sh.never : &sh.bar[warp][stg], injected ? 0u : (it / NSTAGE) & 1,
                             injected ? a.inject_polls : WAIT_POLLS)) {
        // A copy never completed: report it, drain what is still in flight
        // (bounded, at the full limit), and contribute nothing more.
        if (lane == 0) atomicOr(a.c.status, DEV_ERR_TIMEOUT);
        const uint32_t inflight = y == y0 ? min((uint32_t)FirstCopies<G>::N, y1 - y) : min((uint32_t)NSTAGE, y1 - y);
        for (uint32_t q = 0; q < inflight; ++q)
          mbar_wait_bounded(&sh.bar[warp][(it + q) % NSTAGE], ((it + q) / NSTAGE) & 1, WAIT_POLLS);
        it += inflight;   // the ring is empty again, its phases in step
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) { S.m[nt] = -INFINITY; S.l[nt] = 0.f; S.e[nt] = 0.f; }
        return cur;
      }
      if (FirstCopies<G>::N < NSTAGE && y == y0 && y0 + 1 < y1) {   // the ring's second copy
        int nidx, nseg;
        const bool nwin = ic.take(geo, &nidx, &nseg);
        const int s1 = (it + 1) % NSTAGE;
        issue_item<BITS, AFFINE>(a, geo, nseg, wm, nwin, nidx, sh.stage[warp][s1], &sh.bar[warp][s1], lane);
      }
      const unsigned char* st = sh.stage[warp][stg];
      int idx;
      if (cc.take(geo.ni(j), geo.win_chunks(j), &idx)) {
        window_chunk_compute<BITS, G, KEEP>(a, sh, st, idx, j, lane, S, geo.n_win(j));
      } else if ((idx + 1) * PB <= geo.n_packed(j)) {
        packed_block_compute<BITS, G, AFFINE, true, KEEP>(a, sh, st, idx, warp, lane, qb, qscale, qoff, qsum, S,
                                                          geo.n_packed(j));
      } else {
        packed_block_compute<BITS, G, AFFINE, false, KEEP>(a, sh, st, idx, warp, lane, qb, qscale, qoff, qsum, S,
                                                           geo.n_packed(j));
      }
      __syncwarp();
      if (y + NSTAGE < y1) {
        fence_proxy_async();
        int nidx, nseg;
        const bool nwin = ic.take(geo, &nidx, &nseg);
        issue_item<BITS, AFFINE>(a, geo, nseg, wm, nwin, nidx, sh.stage[warp][stg], &sh.bar[warp][stg], lane);
      }
    }
  }
  if constexpr (KEEP) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
      if (S.F[nt] > 0.f) flush_pv(S, nt);
  }
  return cur;
}

// ---- the kernel --------------------------------------------------------------------
// One CTA per SM.  The CTA's stream-K item range is handled in batches of at
// most UMAX unit segments (one batch unless the units are short).  The
// queries of the batch's units are prepared once; warp w streams items
// [x0 + len w / NW, x0 + len (w + 1) / NW) of the batch, crossing a unit
// boundary when its range does; the warps' states are merged per segment
// into the CTA's partial for that unit, and the last CTA to finish a unit
// merges its partials into the output.
// Kernel parameter of the per-sequence token counts (empty when every
// sequence holds the same number of tokens).
template <bool RAGGED> struct RaggedParam {};
template <> struct RaggedParam<true> { RaggedTable t; };

// Item geometry of unit u, and the unit holding global item y.
template <bool RAGGED>
__device__ __forceinline__ SegGeom unit_geom(const DecodeArgs& a, const RaggedParam<RAGGED>& rp, int u) {
  SegGeom g;
  if constexpr (RAGGED) {
    const DevCache& c = a.c;
    const int b = u / c.n_kv_heads, h = u - b * c.n_kv_heads;
    const SeqGeom s = seq_geom(rp.t.n[b], c.sink, c.recent, c.chunk, c.ring_slots);
    g.ni = s.win_chunks + s.pack_blocks;
    g.start = rp.t.item_start[b] + (uint32_t)h * (uint32_t)g.ni;
    g.win_chunks = s.win_chunks; g.n_sink = s.n_sink; g.n_win = s.n_sink + s.n_recent;
    g.n_packed = s.n_packed; g.ring_first = s.ring_first;
  } else {
    g.ni = a.items_per_unit;
    g.start = (uint32_t)u * (uint32_t)a.items_per_unit;
    g.win_chunks = a.win_chunks; g.n_sink = a.n_sink; g.n_win = a.n_sink + a.n_recent;
    g.n_packed = a.n_packed; g.ring_first = a.ring_first;
  }
  return g;
}
template <bool RAGGED>
__device__ __forceinline__ int unit_of(const DecodeArgs& a, const RaggedParam<RAGGED>& rp, uint32_t y) {
  if constexpr (RAGGED) {
    int lo = 0, hi = rp.t.nseq - 1;   // last sequence whose first item is <= y
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (rp.t.item_start[mid] <= y) lo = mid; else hi = mid - 1;
    }
    const DevCache& c = a.c;
    const SeqGeom s = seq_geom(rp.t.n[lo], c.sink, c.recent, c.chunk, c.ring_slots);
    const uint32_t ni = (uint32_t)(s.win_chunks + s.pack_blocks);
    return lo * c.n_kv_heads + (int)((y - rp.t.item_start[lo]) / ni);
  } else {
    return (int)(y / (uint32_t)a.items_per_unit);
  }
}

// Segment geometry of the batch of nseg units from u_first into shared
// memory (threads tid < UMAX; unused slots empty, past the batch's end).
template <bool RAGGED, class SM>
__device__ __forceinline__ void fill_batch_geom(const DecodeArgs& a, const RaggedParam<RAGGED>& rp, SM& sh,
                                                int u_first, int nseg, int tid) {
  if (tid < UMAX) {
    SegGeom g = unit_geom<RAGGED>(a, rp, u_first + min(tid, nseg - 1));
    if (tid >= nseg) { g.start += (uint32_t)g.ni; g.ni = 0; }
    sh.geom[tid] = g;
  }
}

template <int BITS, int G, bool AFFINE, bool RAGGED>
__global__ void __launch_bounds__(Warps<BITS>::N * 32, 1)
    decode_kernel(const __grid_constant__ DecodeArgs a, const __grid_constant__ WindowMaps wm,
                  const __grid_constant__ RaggedParam<RAGGED> rp) {
  constexpr int NW = Warps<BITS>::N;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // stages on 1 KB boundaries (swizzle atoms): the launch adds 1 KB of slack
  Smem<BITS, G>& sh = *reinterpret_cast<Smem<BITS, G>*>(smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u));
  constexpr int NT = (G + 3) / 4;
  constexpr int NG = NT * 4;                 // heads incl. zero padding
  const DevCache& c = a.c;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Hq = c.n_kv_heads * G;
  const uint32_t cta = blockIdx.x;
  const uint32_t X0 = cta_begin(a, cta), X1 = X0 + a.cta_q + (cta < a.cta_r ? 1u : 0u);
  const int U0 = unit_of<RAGGED>(a, rp, X0), U1 = unit_of<RAGGED>(a, rp, X1 - 1);

  // the window maps' descriptors are kernel parameters: fetch them now
  if (tid == 0) {
    prefetch_tensormap(&wm.sink_k); prefetch_tensormap(&wm.sink_v);
    prefetch_tensormap(&wm.ring_k); prefetch_tensormap(&wm.ring_v);
  }
  // each warp initialises its own copy ring's barriers
  if (lane < NSTAGE) {
    mbar_init(&sh.bar[warp][lane], 1);
    if (warp == 0 && lane == 0) mbar_init(&sh.never, 1);
    fence_barrier_init();
  }
  // the first batch's segment geometry depends on the parameters alone
  if constexpr (RAGGED) fill_batch_geom<RAGGED>(a, rp, sh, U0, min(UMAX, U1 - U0 + 1), tid);
  __syncthreads();
  uint32_t it = 0;
  // q' and the cache may come from the kernel launched just before this one
  grid_dependency_wait();
  grid_dependents_may_launch();

  for (int u_first = U0; u_first <= U1; u_first += UMAX) {
    const int nseg = min(UMAX, U1 - u_first + 1);
    const Geo<RAGGED, BITS, G> geo{sh, a, u_first};
    if constexpr (RAGGED) {   // later batches' geometry (the previous batch ended with a barrier)
      if (u_first != U0) {
        fill_batch_geom<RAGGED>(a, rp, sh, u_first, nseg, tid);
        __syncthreads();
      }
    }
    const SegGeom glast = geo(nseg - 1);
    const uint32_t x0 = max(X0, geo(0).start);
    const uint32_t x1 = min(X1, glast.start + (uint32_t)glast.ni);
    const uint32_t len = x1 - x0;
    const uint32_t y0 = x0 + (uint32_t)((uint64_t)len * (uint32_t)warp / NW);
    const uint32_t y1 = x0 + (uint32_t)((uint64_t)len * (uint32_t)(warp + 1) / NW);

    // ---- query loads first (ahead of the copy flood), then the first copies ------
    // pair p = (segment p / NG, head p % NG); warp w takes pairs w, w + NW, ...
    constexpr int PMAX = (UMAX * NG + NW - 1) / NW;
    float4 qv[PMAX];
#pragma unroll
    for (int i = 0; i < PMAX; ++i) {
      const int p = warp + i * NW, pj = p / NG, g = p % NG;
      qv[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (pj < nseg && g < G) {
        const int pu = u_first + pj;
        const int pb = pu / c.n_kv_heads, ph = pu % c.n_kv_heads;
        qv[i] = __ldg(reinterpret_cast<const float4*>(a.q + ((size_t)pb * Hq + (size_t)ph * G + g) * D) + lane);
      }
    }
    // (the previous batch ended with a barrier: its slot reads are complete
    // before these copies land in the stage area)
    GCursor ic;
    warp_items_prefetch<BITS, AFFINE, G>(a, wm, sh, geo, y0, y1, warp, lane, it, ic);
    if (tid < UMAX - 1) sh.bused[tid] = 0;
    if (tid < UMAX * G) sh.segMi[tid / G][tid % G] = float_order(-INFINITY);

    // ---- scaled query: two int8 terms and two fp16 terms per head ----------------
#pragma unroll
    for (int i = 0; i < PMAX; ++i) {
      const int p = warp + i * NW, pj = p / NG, g = p % NG;
      if (pj < nseg) {
        float x[4] = {qv[i].x * a.scale_log2, qv[i].y * a.scale_log2, qv[i].z * a.scale_log2,
                      qv[i].w * a.scale_log2};
        // |x| >= 0 orders like its bit pattern: one integer warp reduction
        const float mx = __uint_as_float(__reduce_max_sync(
            FULL_MASK, __float_as_uint(fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3]))))));
        const float sigma = mx / 127.f;
        const float inv = mx > 0.f ? 127.f / mx : 0.f;
        int sum = 0;
        uint32_t w0 = 0, w1 = 0;
        __half hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float y = x[e] * inv;
          const float t0 = fminf(fmaxf(rintf(y), -127.f), 127.f);
          const float t1 = fminf(fmaxf(rintf((y - t0) * 254.f), -127.f), 127.f);
          w0 |= (uint32_t)(uint8_t)(int8_t)t0 << (8 * e);
          w1 |= (uint32_t)(uint8_t)(int8_t)t1 << (8 * e);
          sum += (int)t0 * 254 + (int)t1;
          hi[e] = __float2half_rn(x[e]);
          lo[e] = __float2half_rn(x[e] - __half2float(hi[e]));
        }
        *reinterpret_cast<uint32_t*>(&sh.qterm[pj][g][0][4 * lane]) = w0;
        *reinterpret_cast<uint32_t*>(&sh.qterm[pj][g][1][4 * lane]) = w1;
        *reinterpret_cast<uint2*>(&sh.qh[pj][g][0][4 * lane]) = *reinterpret_cast<const uint2*>(hi);
        *reinterpret_cast<uint2*>(&sh.qh[pj][g][1][4 * lane]) = *reinterpret_cast<const uint2*>(lo);
        sum = __reduce_add_sync(FULL_MASK, sum);
        if (lane == 0) {
          sh.qscale[pj][g] = sigma / 254.f;
          sh.qsum[pj][g] = (sigma / 254.f) * (float)sum;
        }
      }
    }
    __syncthreads();

    // ---- this warp's items -----------------------------------------------------------
    SoftmaxState<NT> S;
    const int jl = warp_run<BITS, G, AFFINE>(a, wm, sh, geo, y0, y1, warp, lane, it, ic, S);
    // The warp's ring has drained: its final state goes into its own stages
    // (an idle warp's slot, maximum and sum are neutral: every slot is read
    // below, with weight 0 where the warp is not a member).
    if (jl >= 0) {
      state_to_slot<BITS, G, AFFINE>(S, warp_slot(sh, warp), sh.sm[warp], sh.sl[warp], lane);
      raise_segment_max(sh, jl, S.m, lane);
    } else {
      for (int e = lane; e < G * D; e += 32) warp_slot(sh, warp)[e / D][e % D] = 0.f;
      if (lane < G) { sh.sm[warp][lane] = -INFINITY; sh.sl[warp][lane] = 0.f; }
    }
    if (lane == 0) sh.wseg[warp] = jl;
    __syncthreads();

    // ---- merge weights: thread (segment j, warp w, head g) --------------------------
    for (int t = tid; t < UMAX * NW * G; t += NW * 32) {
      const int j = t / (NW * G), w = (t / G) % NW, g = t % G;
      sh.wf[j][w][g] = (j < nseg && sh.wseg[w] == j)
                           ? merge_weight(sh.sm[w][g], order_float(sh.segMi[j][g])) : 0.f;
      if (t < (UMAX - 1) * G) {
        const int jb = t / G, gb = t % G;
        sh.bf[jb][gb] = (jb < nseg - 1 && sh.bused[jb])
                            ? merge_weight(sh.bm[jb][gb], order_float(sh.segMi[jb][gb])) : 0.f;
      }
    }
    if (tid < nseg) {   // arrivals before the last one (0: the unit lies in this CTA alone;
                        // -1: the unit has no tokens)
      const SegGeom g = geo(tid);
      const int o = (int)(cta_of(a, g.start + (uint32_t)g.ni - 1) - cta_of(a, g.start));
      if constexpr (RAGGED) sh.others[tid] = g.ni == 0 ? -1 : o;
      else sh.others[tid] = o;
    }
    __syncthreads();

    // ---- weighted sums: thread (head g, dim d), the slots in two halves of
    // independent loads.  Segments that other CTAs also hold are published
    // straight away.
    constexpr int NH = (NW + 1) / 2;
    for (int e = tid; e < G * D; e += NW * 32) {
      const int g = e / D, d = e % D;
      float Oj[UMAX];
#pragma unroll
      for (int jj = 0; jj < UMAX; ++jj)
        Oj[jj] = (jj < nseg - 1 && sh.bused[jj]) ? sh.bf[jj][g] * sh.bo[jj][g][d] : 0.f;
#pragma unroll
      for (int h0 = 0; h0 < NW; h0 += NH) {
        float x[NH];
#pragma unroll
        for (int w = 0; w < NH; ++w) x[w] = h0 + w < NW ? warp_slot(sh, h0 + w)[g][d] : 0.f;
#pragma unroll
        for (int jj = 0; jj < UMAX; ++jj) {
          if (jj < nseg) {
#pragma unroll
            for (int w = 0; w < NH; ++w)
              if (h0 + w < NW) Oj[jj] = fmaf(sh.wf[jj][h0 + w][g], x[w], Oj[jj]);
          }
        }
      }
#pragma unroll
      for (int jj = 0; jj < UMAX; ++jj) {
        if (jj >= nseg) break;
        const bool has_b = jj < nseg - 1 && sh.bused[jj];
        const float O = Oj[jj];
        segment_sum(sh, jj)[g][d] = O;
        float L = 0.f;
        if (d == 0) {
          L = has_b ? sh.bf[jj][g] * sh.bl[jj][g] : 0.f;
#pragma unroll
          for (int w = 0; w < NW; ++w) L = fmaf(sh.wf[jj][w][g], sh.sl[w][g], L);
          sh.segL[jj][g] = L;
        }
        if (sh.others[jj] > 0) {
          const int uu = u_first + jj;
          const uint32_t slot = cta - cta_of(a, geo(jj).start);
          if (slot < (uint32_t)c.max_splits) {
            float* part = a.partials + (((size_t)uu * c.max_splits + slot) * G + g) * PART;
            part[d] = O;
            if (d == 0) { part[D] = order_float(sh.segMi[jj][g]); part[D + 1] = L; }
          } else if (e == 0) {
            atomicOr(c.status, DEV_ERR_SPLITS);   // the host's split bound was wrong: never write past it
          }
        }
      }
    }

    // ---- arrival: the last CTA of a unit merges its partials -----------------------
    // The barrier orders every thread's partial writes before the acq_rel
    // atomics, which publish them at gpu scope (release) and, for the last
    // arrival, make the other CTAs' partials visible (acquire).
    __syncthreads();
    if (tid < nseg) {
      int last = sh.others[tid] >= 0;   // a unit without tokens has no output
      if (sh.others[tid] > 0) {
        const int uu = u_first + tid;
        int prevc;
        asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;\n"
                     : "=r"(prevc) : "l"(a.counters + (size_t)uu * c.counter_stride) : "memory");
        last = prevc == sh.others[tid];
      }
      sh.is_last[tid] = last;
    }
    __syncthreads();
    // one warp per (segment, head) of the units this CTA completes
    for (int p = warp; p < nseg * G; p += NW) {
      const int jj = p / G, g = p % G;
      if (!sh.is_last[jj]) continue;
      const int uu = u_first + jj;
      const int bb = uu / c.n_kv_heads, hh = uu % c.n_kv_heads;
      float* dst = a.out + ((size_t)bb * Hq + (size_t)hh * G + g) * D + 4 * lane;
      if (sh.others[jj] == 0) {   // the whole unit lies in this CTA
        const float4 O = reinterpret_cast<const float4*>(segment_sum(sh, jj)[g])[lane];
        const float il = 1.f / sh.segL[jj][g];
        *reinterpret_cast<float4*>(dst) = make_float4(O.x * il, O.y * il, O.z * il, O.w * il);
        continue;
      }
      const int nparts = min(sh.others[jj] + 1, c.max_splits);
      const float* pbase = a.partials + (size_t)uu * c.max_splits * G * PART + (size_t)g * PART;
      float M = -INFINITY, L = 0.f;
      float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
      // the partials in index order, in rounds of eight with all loads of a
      // round in flight at once; the running (M, L, O) is rescaled when a
      // round raises M
      for (int sp0 = 0; sp0 < nparts; sp0 += 8) {
        float4 v[8];
        float mw[8], lw[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const bool ok = sp0 + q < nparts;
          const float* part = pbase + (size_t)(ok ? sp0 + q : 0) * G * PART;
          v[q] = ok ? __ldcg(reinterpret_cast<const float4*>(part) + lane) : make_float4(0.f, 0.f, 0.f, 0.f);
          mw[q] = ok ? __ldcg(part + D) : -INFINITY;
          lw[q] = ok ? __ldcg(part + D + 1) : 0.f;
        }
        float Mr = M;
#pragma unroll
        for (int q = 0; q < 8; ++q) Mr = fmaxf(Mr, mw[q]);
        const float fr = merge_weight(M, Mr);
        L *= fr;
        O.x *= fr; O.y *= fr; O.z *= fr; O.w *= fr;
        M = Mr;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float f = merge_weight(mw[q], M);
          L = fmaf(lw[q], f, L);
          O.x = fmaf(v[q].x, f, O.x); O.y = fmaf(v[q].y, f, O.y);
          O.z = fmaf(v[q].z, f, O.z); O.w = fmaf(v[q].w, f, O.w);
        }
      }
      const float il = 1.f / L;
      *reinterpret_cast<float4*>(dst) = make_float4(O.x * il, O.y * il, O.z * il, O.w * il);
    }
    if (tid < nseg && sh.is_last[tid]) a.counters[(size_t)(u_first + tid) * c.counter_stride] = 0;
    __syncthreads();
    fence_proxy_async();  // the stage area was written as slots; the next batch's copies overwrite it
  }
}

template <int BITS, int G, bool AFFINE, bool RAGGED>
cudaError_t launch_t(const DecodeArgs& a, const WindowMaps& wm, const RaggedTable* rt, cudaStream_t s) {
  auto k = decode_kernel<BITS, G, AFFINE, RAGGED>;
  static_assert(sizeof(Smem<BITS, G>) + 1024 <= 232448, "decode shared memory above the per-CTA limit");
  const int smem = (int)sizeof(Smem<BITS, G>) + 1024;
  static int attr_done[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    attr_done[dev] = 1;
  }
  RaggedParam<RAGGED> rp;
  if constexpr (RAGGED) rp.t = *rt;
  return launch_with_overlap(k, dim3((unsigned)a.grid), dim3(Warps<BITS>::N * 32), (size_t)smem, s, a, wm, rp);
}

template <int BITS, int G, bool AFFINE>
cudaError_t launch_r(const DecodeArgs& a, const WindowMaps& wm, const RaggedTable* rt, cudaStream_t s) {
  return rt ? launch_t<BITS, G, AFFINE, true>(a, wm, rt, s) : launch_t<BITS, G, AFFINE, false>(a, wm, rt, s);
}

template <int BITS, bool AFFINE>
cudaError_t launch_g(const DecodeArgs& a, const WindowMaps& wm, const RaggedTable* rt, cudaStream_t s) {
  switch (a.c.group) {
    case 1: return launch_r<BITS, 1, AFFINE>(a, wm, rt, s);
    case 2: return launch_r<BITS, 2, AFFINE>(a, wm, rt, s);
    case 4: return launch_r<BITS, 4, AFFINE>(a, wm, rt, s);
    case 8: return launch_r<BITS, 8, AFFINE>(a, wm, rt, s);
    default: return cudaErrorInvalidValue;
  }
}

template <int BITS, int G, bool AFFINE>
int occupancy_t() {
  auto k = decode_kernel<BITS, G, AFFINE, false>;
  const int smem = (int)sizeof(Smem<BITS, G>) + 1024;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return 1;
  int n = 0;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, Warps<BITS>::N * 32, smem);
  return n > 0 ? n : 1;
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, const WindowMaps& wm, const RaggedTable* rt, cudaStream_t s) {
  const bool affine = a.c.quantizer == WUSHKV_AFFINE_PCTCLIP;
  switch (a.c.bits) {
    case 2: return affine ? launch_g<2, true>(a, wm, rt, s) : launch_g<2, false>(a, wm, rt, s);
    case 3: return affine ? launch_g<3, true>(a, wm, rt, s) : launch_g<3, false>(a, wm, rt, s);
    case 4: return affine ? launch_g<4, true>(a, wm, rt, s) : launch_g<4, false>(a, wm, rt, s);
    default: return cudaErrorInvalidValue;
  }
}

// Resident CTAs per SM of the decode kernel for this configuration (the
// grid fills one wave).
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
