// Host side of the libwushkv C ABI: configuration checks, cache layout, the
// window/flush bookkeeping of each append, decode split policy, export and
// status.  See include/wushkv.h for the contract of every entry point.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include "wushkv_internal.cuh"

struct wushkv_cache {
  wushkv_config cfg;
  wushkv_layout lay;
  uint8_t* base;
  size_t bytes;
  std::vector<int64_t> seq_n;   // tokens of each sequence
  bool uniform;                 // every sequence holds n tokens
  int64_t n;
  double alpha;     // QuEST clip ratio in use
  wushkv::WindowMaps wmaps;   // tensor maps over the fp16 windows (decode)
  const int32_t* page_table;  // paged caches: the caller's page table (device), row stride pt_stride
  int32_t pt_stride;
  mutable wushkv::RaggedTable rt;   // the ragged decode's kernel parameter, rebuilt per call
};

namespace {

using namespace wushkv;

// Decode work split: each unit's cache is a sequence of items of about 4 KB
// (window chunks of 8 fp16 tokens spread among packed blocks of 64 tokens);
// the units' items are shared equally among the CTAs of one wave
// (stream-K), at least MIN_CTA_ITEMS each.  Each CTA touching a unit writes
// one partial; the workspace holds max(3, MAX_GRID / units + 2) partials
// per unit and the grid shrinks until no unit can meet more CTAs than that.
constexpr int WIN_CHUNK = 8;
constexpr int PACK_BLOCK = 64;
constexpr int64_t MIN_CTA_ITEMS = 8;
constexpr int MAX_GRID = 2048;
// The unit-merging CTA stages the (m, l) of all partials of a unit in its
// shared memory; at most this many partials per unit.
constexpr int MAX_PARTS_PER_UNIT = 256;
// Appends with at least this many new tokens per unit (from the first
// quad boundary) take the tensor-core kernel (two 128-token tiles).
constexpr int64_t TC_MIN_TOKENS = 256;
constexpr int64_t TC_MIN_CTA_TILES = 6;
// Each unit's arrival counter sits on its own 128-byte line, so that the
// atomics of different units at the end of a decode do not queue on one line.
constexpr size_t COUNTER_BYTES = 128;
// Fault injection for tests (wushkv_inject_decode_timeout): 0 = off.
std::atomic<uint32_t> g_inject_polls{0};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int64_t packed_count(int64_t n, const wushkv_config& c) {
  const int64_t ns = n < c.sink ? n : c.sink;
  const int64_t m = n - ns;
  return (m >= (int64_t)c.recent + c.chunk) ? (int64_t)c.chunk * ((m - c.recent) / c.chunk) : 0;
}

// ---- default QuEST clip ratio ------------------------------------------------
// The clip ratio that minimises the mean squared error of the 2^b-level
// mid-rise uniform quantiser on a unit Gaussian (Max, 1960), found as the
// zero of the derivative of that error with respect to the clip ratio.  The
// derivative only involves the moving levels c_i = (2i + 1) alpha / L:
//   dMSE/dalpha = -2 sum_i (2i + 1)/L * int_{cell i} (x - c_i) phi(x) dx.
double std_pdf(double x) { return std::isinf(x) ? 0.0 : std::exp(-0.5 * x * x) * 0.3989422804014327; }
double std_cdf(double x) {
  if (std::isinf(x)) return x > 0 ? 1.0 : 0.0;
  return 0.5 * std::erfc(-x * 0.7071067811865476);
}
double mse_slope(double alpha, int L) {
  const double step = 2.0 * alpha / L;
  double acc = 0.0;
  for (int i = -L / 2; i < L / 2; ++i) {
    const double lo = (i == -L / 2) ? -INFINITY : i * step;
    const double hi = (i == L / 2 - 1) ? INFINITY : (i + 1) * step;
    const double ci = (i + 0.5) * step;
    const double first = (std_pdf(lo) - std_pdf(hi)) - ci * (std_cdf(hi) - std_cdf(lo));
    acc += -2.0 * (2.0 * i + 1.0) / L * first;
  }
  return acc;
}
double gaussian_optimal_alpha(int bits) {
  const int L = 1 << bits;
  double lo = 0.25, hi = 16.0;
  for (int it = 0; it < 200; ++it) {
    const double mid = 0.5 * (lo + hi);
    if (mid == lo || mid == hi) break;
    if (mse_slope(mid, L) < 0) lo = mid; else hi = mid;
  }
  return 0.5 * (lo + hi);
}

// ---- configuration + layout ----------------------------------------------------
wushkv_status check_config(const wushkv_config* c) {
  if (!c) return WUSHKV_EINVAL;
  if (c->batch < 1 || c->n_kv_heads < 1 || c->n_q_heads < 1 || c->max_ctx < 1) return WUSHKV_EINVAL;
  if (c->n_q_heads % c->n_kv_heads) return WUSHKV_EINVAL;
  const int G = c->n_q_heads / c->n_kv_heads;
  if (c->head_dim != 128) return WUSHKV_EUNSUPPORTED;
  if (G != 1 && G != 2 && G != 4 && G != 8) return WUSHKV_EUNSUPPORTED;
  if (c->bits < 2 || c->bits > 4) return WUSHKV_EUNSUPPORTED;
  if (c->quantizer != WUSHKV_QUEST_INT && c->quantizer != WUSHKV_AFFINE_PCTCLIP) return WUSHKV_EINVAL;
  if (c->sink < 0 || c->recent < 0 || c->chunk < 4) return WUSHKV_EINVAL;
  if (c->sink % 4 || c->chunk % 4) return WUSHKV_EUNSUPPORTED;
  if (c->quantizer == WUSHKV_QUEST_INT) {
    if (c->quest_alpha < 0 || c->quest_alpha > (double)(1 << (c->bits - 1)) ||
        std::isnan(c->quest_alpha))
      return WUSHKV_EINVAL;
  } else {
    if (c->clip_lo_rank < 1 || c->clip_hi_rank > 128 || c->clip_lo_rank >= c->clip_hi_rank)
      return WUSHKV_EINVAL;
    if (c->clip_lo_rank > 8 || c->clip_hi_rank < 121) return WUSHKV_EUNSUPPORTED;
  }
  if ((int64_t)c->batch * c->n_kv_heads > 65535) return WUSHKV_EUNSUPPORTED;
  if (c->num_pages < 0) return WUSHKV_EINVAL;
  return WUSHKV_OK;
}

int max_splits_for(const wushkv_config& c, int packed_capacity) {
  (void)packed_capacity;
  const int units = c.batch * c.n_kv_heads;
  const int ms = MAX_GRID / units + 2;
  return ms < 3 ? 3 : (ms > MAX_PARTS_PER_UNIT ? MAX_PARTS_PER_UNIT : ms);
}

// Bytes of the packed region: per unit its block records, or the page
// pool (num_pages + 1 pages: the last one is the spare page that
// out-of-range page ids are sent to).
size_t packed_region_bytes(const wushkv_config& c, const wushkv_layout& L) {
  if (c.num_pages > 0) return (size_t)(c.num_pages + 1) * L.page_bytes;
  return (size_t)c.batch * c.n_kv_heads * L.unit_stride;
}

void make_layout(const wushkv_config& c, wushkv_layout* L) {
  std::memset(L, 0, sizeof(*L));
  const size_t U = (size_t)c.batch * c.n_kv_heads;
  const int G = c.n_q_heads / c.n_kv_heads;
  if (c.bits == 3) { L->n_planes = 2; L->plane_bits[0] = 2; L->plane_bits[1] = 1; }
  else { L->n_planes = 1; L->plane_bits[0] = c.bits; }
  L->packed_capacity = (int)align_up((size_t)c.max_ctx, 128);
  L->meta_bytes = c.quantizer == WUSHKV_QUEST_INT ? 2 : 4;
  // block record of 64 packed tokens: K planes, V planes, K meta, V meta
  size_t in_block = 0;
  for (int p = 0; p < L->n_planes; ++p) { L->k_plane_off[p] = in_block; in_block += 64 * 16 * L->plane_bits[p]; }
  for (int p = 0; p < L->n_planes; ++p) { L->v_plane_off[p] = in_block; in_block += 64 * 16 * L->plane_bits[p]; }
  L->k_meta_off = in_block; in_block += 64 * L->meta_bytes;
  L->v_meta_off = in_block; in_block += 64 * L->meta_bytes;
  L->block_stride = in_block;                                   // a multiple of 128
  L->unit_stride = (size_t)(L->packed_capacity / 64) * L->block_stride;
  if (c.num_pages > 0) {   // pages of n_kv_heads block records, one spare page at the end
    L->num_pages = c.num_pages;
    L->page_bytes = (size_t)c.n_kv_heads * L->block_stride;
  }
  // every region is followed by a guard band (see guard_spans)
  size_t off = align_up(packed_region_bytes(c, *L) + WUSHKV_GUARD_BYTES, 256);   // packed region at offset 0
  L->sink_unit_stride = (size_t)c.sink * 128 * 2;
  L->sink_k_off = off; off = align_up(off + U * L->sink_unit_stride + WUSHKV_GUARD_BYTES, 256);
  L->sink_v_off = off; off = align_up(off + U * L->sink_unit_stride + WUSHKV_GUARD_BYTES, 256);
  L->ring_slots = c.recent + c.chunk;
  L->ring_unit_stride = (size_t)L->ring_slots * 128 * 2;
  L->ring_k_off = off; off = align_up(off + U * L->ring_unit_stride + WUSHKV_GUARD_BYTES, 256);
  L->ring_v_off = off; off = align_up(off + U * L->ring_unit_stride + WUSHKV_GUARD_BYTES, 256);
  const int ms = max_splits_for(c, L->packed_capacity);
  L->workspace_off = off;
  L->workspace_bytes = align_up(U * (size_t)ms * G * PARTIAL_FLOATS * sizeof(float), COUNTER_BYTES) +
                       U * COUNTER_BYTES;
  off = align_up(off + L->workspace_bytes + WUSHKV_GUARD_BYTES, 256);
  L->status_off = off; off = align_up(off + 256, 256);
  L->total_bytes = off;
}

// Start offsets of the guard bands that follow the packed region, sink K,
// sink V, ring K, ring V and the workspace.
void guard_spans(const wushkv_config& c, const wushkv_layout& L, size_t out[6]) {
  const size_t U = (size_t)c.batch * c.n_kv_heads;
  out[0] = packed_region_bytes(c, L);
  out[1] = L.sink_k_off + U * L.sink_unit_stride;
  out[2] = L.sink_v_off + U * L.sink_unit_stride;
  out[3] = L.ring_k_off + U * L.ring_unit_stride;
  out[4] = L.ring_v_off + U * L.ring_unit_stride;
  out[5] = L.workspace_off + L.workspace_bytes;
}

DevCache dev_view(const wushkv_cache* h) {
  const wushkv_config& c = h->cfg;
  const wushkv_layout& L = h->lay;
  DevCache d;
  std::memset(&d, 0, sizeof(d));
  for (int p = 0; p < L.n_planes; ++p) {
    d.k_plane[p] = h->base + L.k_plane_off[p];
    d.v_plane[p] = h->base + L.v_plane_off[p];
    d.plane_bits[p] = L.plane_bits[p];
  }
  d.n_planes = L.n_planes;
  d.bits = c.bits;
  d.quantizer = c.quantizer;
  d.k_meta = h->base + L.k_meta_off;
  d.v_meta = h->base + L.v_meta_off;
  d.meta_bytes = (int)L.meta_bytes;
  d.unit_stride = L.unit_stride;
  d.block_stride = L.block_stride;
  d.sink_k = reinterpret_cast<__half*>(h->base + L.sink_k_off);
  d.sink_v = reinterpret_cast<__half*>(h->base + L.sink_v_off);
  d.ring_k = reinterpret_cast<__half*>(h->base + L.ring_k_off);
  d.ring_v = reinterpret_cast<__half*>(h->base + L.ring_v_off);
  d.sink = c.sink; d.recent = c.recent; d.chunk = c.chunk; d.ring_slots = L.ring_slots;
  d.packed_capacity = L.packed_capacity;
  d.max_splits = max_splits_for(c, L.packed_capacity);
  const size_t U = (size_t)c.batch * c.n_kv_heads;
  d.partials = reinterpret_cast<float*>(h->base + L.workspace_off);
  d.counters = reinterpret_cast<int*>(h->base + L.workspace_off +
                                      align_up(U * (size_t)d.max_splits * (c.n_q_heads / c.n_kv_heads) *
                                                   PARTIAL_FLOATS * sizeof(float),
                                               COUNTER_BYTES));
  d.counter_stride = (int)(COUNTER_BYTES / sizeof(int));
  d.status = reinterpret_cast<int*>(h->base + L.status_off);
  d.units = (int)U;
  d.n_kv_heads = c.n_kv_heads;
  d.group = c.n_q_heads / c.n_kv_heads;
  d.alpha = h->alpha;
  d.r_lo = c.clip_lo_rank;
  d.r_hi = c.clip_hi_rank;
  d.page_table = c.num_pages > 0 ? h->page_table : nullptr;
  d.pt_stride = h->pt_stride;
  d.num_pages = c.num_pages;
  return d;
}

// The batch-1 view of sequence b used by its own append launches: every
// per-unit region starts at the sequence's first unit.
DevCache seq_view(const wushkv_cache* h, int b) {
  DevCache d = dev_view(h);
  const size_t u0 = (size_t)b * d.n_kv_heads;
  if (d.page_table == nullptr) {
    for (int p = 0; p < d.n_planes; ++p) {
      d.k_plane[p] += u0 * d.unit_stride;
      d.v_plane[p] += u0 * d.unit_stride;
    }
    d.k_meta += u0 * d.unit_stride;
    d.v_meta += u0 * d.unit_stride;
  } else {
    d.page_table += (size_t)b * d.pt_stride;
  }
  d.sink_k += u0 * d.sink * D;
  d.sink_v += u0 * d.sink * D;
  d.ring_k += u0 * d.ring_slots * D;
  d.ring_v += u0 * d.ring_slots * D;
  d.units = d.n_kv_heads;
  return d;
}

wushkv_status cuda_status(cudaError_t e) { return e == cudaSuccess ? WUSHKV_OK : WUSHKV_ECUDA; }

bool valid_dtype(int32_t d) { return d == WUSHKV_F16 || d == WUSHKV_BF16 || d == WUSHKV_F32; }

// Fill the decode arguments of the cache's current state: window/packed
// counts and the split plan.  Returns false if the cache is empty.
int device_sms() {
  static int sms[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 148;
  if (!sms[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    sms[dev] = n;
  }
  return sms[dev];
}

// Most CTAs of a stream-K split that touch one unit: every CTA takes at
// least items / grid items, so a unit of ni items meets at most
// ceil((ni - 1) / q) + 1 of them.
int64_t parts_per_unit_bound(int64_t items, int64_t grid, int64_t ni) {
  const int64_t q = items / grid;
  return (ni - 1 + q - 1) / q + 1;
}

// Fill the decode arguments of the cache's current state: window/packed
// counts and the split plan.  EINVAL if the cache is empty, EUNSUPPORTED if
// the item indices would not fit the kernel's 32-bit arithmetic.
// Fill the decode arguments of the cache's current state: window/packed
// counts and the split plan.  For sequences of unequal lengths *rt is set to
// the cache's table of per-sequence counts and item offsets (else null).
// EINVAL if every sequence is empty, EUNSUPPORTED if the item indices would
// not fit the kernel's 32-bit arithmetic or a ragged batch is too large.
wushkv_status plan_decode(const wushkv_cache* h, const float* q, float* out, float scale, DecodeArgs* a,
                          const RaggedTable** rt) {
  const wushkv_config& c = h->cfg;
  std::memset(a, 0, sizeof(*a));
  *rt = nullptr;
  a->c = dev_view(h);
  if (c.num_pages > 0 && h->page_table == nullptr) return WUSHKV_EINVAL;
  a->q = q;
  a->out = out;
  const float sc = scale > 0.f ? scale : 0.08838834764831845f;  // 1/sqrt(128)
  a->scale_log2 = sc * 1.4426950408889634f;
  const int W = c.recent + c.chunk;
  const int64_t units = a->c.units;
  int64_t items = 0, ni_max = 0, wc_max = 0;
  // Uniform dense caches take the decode variant that reads the geometry
  // from its arguments and addresses the packed region directly; ragged or
  // paged ones the variant with the per-sequence table (and page lookups).
  if (h->uniform && c.num_pages == 0) {
    const int64_t n = h->n;
    if (n == 0) return WUSHKV_EINVAL;
    const SeqGeom g = seq_geom(n, c.sink, c.recent, c.chunk, W);
    a->n_sink = g.n_sink;
    a->n_packed = g.n_packed;
    a->n_recent = g.n_recent;
    a->ring_first = g.ring_first;
    a->win_chunks = g.win_chunks;
    a->pack_blocks = g.pack_blocks;
    ni_max = (int64_t)g.win_chunks + g.pack_blocks;
    wc_max = g.win_chunks;
    items = units * ni_max;
    a->items_per_unit = (int)ni_max;
  } else {
    if (c.batch > MAX_RAGGED_SEQS) return WUSHKV_EUNSUPPORTED;
    RaggedTable& t = h->rt;
    t.nseq = c.batch;
    for (int b = 0; b < c.batch; ++b) {
      const SeqGeom g = seq_geom(h->seq_n[b], c.sink, c.recent, c.chunk, W);
      const int64_t ni = (int64_t)g.win_chunks + g.pack_blocks;
      if (items >= (int64_t(1) << 31)) return WUSHKV_EUNSUPPORTED;
      t.item_start[b] = (uint32_t)items;
      t.n[b] = (int32_t)h->seq_n[b];
      items += (int64_t)c.n_kv_heads * ni;
      if (ni > ni_max) ni_max = ni;
      if (g.win_chunks > wc_max) wc_max = g.win_chunks;
    }
    t.item_start[c.batch] = (uint32_t)(items < (int64_t(1) << 32) ? items : 0);
    if (items == 0) return WUSHKV_EINVAL;
    *rt = &t;
  }
  if (items >= (int64_t(1) << 31) || ni_max * wc_max >= (int64_t(1) << 32)) return WUSHKV_EUNSUPPORTED;
  static int occ[5][9][2] = {};
  int& o = occ[c.bits][a->c.group][c.quantizer];
  if (!o) {
    o = decode_ctas_per_sm(c.bits, a->c.group, c.quantizer);
    if (o <= 0) o = 1;
  }
  int64_t grid = (int64_t)device_sms() * o;
  if (grid > items / MIN_CTA_ITEMS) grid = items / MIN_CTA_ITEMS;
  if (grid > (int64_t)(a->c.max_splits - 1) * units) grid = (int64_t)(a->c.max_splits - 1) * units;
  if (grid < 1) grid = 1;
  while (grid > 1 && parts_per_unit_bound(items, grid, ni_max) > a->c.max_splits) --grid;
  a->grid = (int)grid;
  a->cta_q = (uint32_t)(items / grid);
  a->cta_r = (uint32_t)(items % grid);
  a->partials = a->c.partials;
  a->counters = a->c.counters;
  a->inject_polls = g_inject_polls.load(std::memory_order_relaxed);
  return WUSHKV_OK;
}

}  // namespace

extern "C" {

double wushkv_default_quest_alpha(int32_t bits) {
  if (bits < 2 || bits > 4) return 0.0;
  static double cached[5] = {0, 0, 0, 0, 0};
  if (cached[bits] == 0.0) cached[bits] = gaussian_optimal_alpha(bits);
  return cached[bits];
}

const char* wushkv_strerror(int32_t s) {
  switch (s) {
    case WUSHKV_OK: return "ok";
    case WUSHKV_EINVAL: return "invalid argument";
    case WUSHKV_ECAPACITY: return "cache capacity exceeded";
    case WUSHKV_EUNSUPPORTED: return "unsupported configuration";
    case WUSHKV_ECUDA: return "CUDA error";
    default: return "unknown status";
  }
}

size_t wushkv_cache_bytes(const wushkv_config* cfg) {
  if (check_config(cfg) != WUSHKV_OK) return 0;
  wushkv_layout L;
  make_layout(*cfg, &L);
  return L.total_bytes;
}

wushkv_status wushkv_cache_create(const wushkv_config* cfg, void* dev_mem, size_t bytes,
                                  void* stream, wushkv_cache** out) {
  if (!out) return WUSHKV_EINVAL;
  *out = nullptr;
  const wushkv_status st = check_config(cfg);
  if (st != WUSHKV_OK) return st;
  if (!dev_mem || (reinterpret_cast<uintptr_t>(dev_mem) & 255)) return WUSHKV_EINVAL;
  wushkv_layout L;
  make_layout(*cfg, &L);
  if (bytes < L.total_bytes) return WUSHKV_EINVAL;
  wushkv_cache* h = new (std::nothrow) wushkv_cache;
  if (!h) return WUSHKV_EINVAL;
  h->cfg = *cfg;
  h->lay = L;
  h->base = static_cast<uint8_t*>(dev_mem);
  h->bytes = bytes;
  h->n = 0;
  h->seq_n.assign((size_t)cfg->batch, 0);
  h->uniform = true;
  h->page_table = nullptr;
  h->pt_stride = 0;
  h->alpha = cfg->quest_alpha > 0 ? cfg->quest_alpha : wushkv_default_quest_alpha(cfg->bits);
  make_window_maps(dev_view(h), &h->wmaps);
  cudaError_t e = cudaMemsetAsync(dev_mem, 0, L.total_bytes, static_cast<cudaStream_t>(stream));
  size_t guards[6];
  guard_spans(*cfg, L, guards);
  for (int i = 0; i < 6 && e == cudaSuccess; ++i)
    e = cudaMemsetAsync(static_cast<uint8_t*>(dev_mem) + guards[i], WUSHKV_GUARD_FILL, WUSHKV_GUARD_BYTES,
                        static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) { delete h; return WUSHKV_ECUDA; }
  *out = h;
  return WUSHKV_OK;
}

wushkv_status wushkv_cache_destroy(wushkv_cache* cache) {
  delete cache;
  return WUSHKV_OK;
}

wushkv_status wushkv_cache_layout(const wushkv_cache* cache, wushkv_layout* out) {
  if (!cache || !out) return WUSHKV_EINVAL;
  *out = cache->lay;
  return WUSHKV_OK;
}

wushkv_status wushkv_cache_tokens(const wushkv_cache* cache, int64_t* n_tokens, int64_t* n_sink,
                                  int64_t* n_packed, int64_t* n_recent) {
  return wushkv_sequence_tokens(cache, 0, n_tokens, n_sink, n_packed, n_recent);
}

wushkv_status wushkv_sequence_tokens(const wushkv_cache* cache, int32_t seq, int64_t* n_tokens, int64_t* n_sink,
                                     int64_t* n_packed, int64_t* n_recent) {
  if (!cache || seq < 0 || seq >= cache->cfg.batch) return WUSHKV_EINVAL;
  const int64_t n = cache->seq_n[seq];
  const int64_t ns = n < cache->cfg.sink ? n : cache->cfg.sink;
  const int64_t P = packed_count(n, cache->cfg);
  if (n_tokens) *n_tokens = n;
  if (n_sink) *n_sink = ns;
  if (n_packed) *n_packed = P;
  if (n_recent) *n_recent = n - ns - P;
  return WUSHKV_OK;
}

}  // extern "C"

namespace {

// Launch plan of one append: FMA-kernel quad ranges (one, or two when new
// tokens reuse ring slots that old flushed tokens are read from) and the
// optional tensor-core bulk kernel.
struct AppendPlan {
  AppendArgs a;
  int64_t range[2][2];
  int nranges;
  bool tc;
  PrefillArgs pf;
  int64_t n1;
};

// Per-CTA quad count of an FMA-kernel range: enough CTAs to fill the GPU,
// up to 64 quads (256 tokens) per CTA.
void set_quad_range(AppendArgs& a, int64_t qa, int64_t qb) {
  a.quad_begin = qa;
  a.n_quads = qb - qa;
  int64_t per = (a.n_quads * a.c.units) / 1184;
  if (per < 1) per = 1;
  if (per > 64) per = 64;
  a.quads_per_cta = (int)per;
}

wushkv_status check_append_args(const wushkv_cache* cache, const void* k_rope_dev, const void* v_dev,
                                int32_t in_dtype, const float* T_k_dev, int32_t bits, int32_t quantizer) {
  if (!cache || !k_rope_dev || !v_dev || !valid_dtype(in_dtype)) return WUSHKV_EINVAL;
  if (reinterpret_cast<uintptr_t>(T_k_dev) & 15) return WUSHKV_EINVAL;  // read as float4
  const wushkv_config& c = cache->cfg;
  if (bits != c.bits || quantizer != c.quantizer) return WUSHKV_EINVAL;
  if (c.num_pages > 0 && cache->page_table == nullptr) return WUSHKV_EINVAL;
  return WUSHKV_OK;
}

size_t dtype_bytes(int32_t dtype) { return dtype == WUSHKV_F32 ? 4 : 2; }

// Plan the append of n_tok tokens to every sequence of `view` (the whole
// cache, or one sequence's batch-1 view), all holding n0 tokens.
void plan_append_view(const wushkv_cache* cache, const DevCache& view, int batch, int64_t n0, int32_t n_tok,
                      const void* k_rope_dev, const void* v_dev, int32_t in_dtype, const float* T_k_dev,
                      AppendPlan* p) {
  const wushkv_config& c = cache->cfg;
  std::memset(p, 0, sizeof(*p));
  const int64_t n1 = n0 + n_tok;
  p->n1 = n1;
  if (n_tok == 0) return;
  const int64_t S = c.sink, W = c.recent + c.chunk;
  const int64_t P0 = packed_count(n0, c), P1 = packed_count(n1, c);

  AppendArgs& a = p->a;
  a.c = view;
  a.k = k_rope_dev;
  a.v = v_dev;
  a.dtype = in_dtype;
  a.T = T_k_dev;
  a.n_tok = n_tok;
  a.n0 = n0;
  a.packed0 = P0;
  a.packed1 = P1;

  // Old recent tokens that this append flushes: [S + P0, min(S + P1, n0)).
  const int64_t flush_end = (S + P1 < n0) ? S + P1 : n0;
  const bool has_old_flush = (P1 > P0) && (S + P0 < n0);
  const int64_t first = has_old_flush ? S + P0 : n0;
  const int64_t q_begin = first / 4, q_end = (n1 + 3) / 4;

  // A bf16 block with a transform goes to the tensor-core key kernel and the
  // value kernel from the first quad boundary at or after n0 to the end;
  // the FMA kernel keeps the flush of old ring rows and the partial quad.
  const int64_t ta = (n0 + 3) / 4 * 4;
  const uintptr_t kv_addr = reinterpret_cast<uintptr_t>(k_rope_dev) | reinterpret_cast<uintptr_t>(v_dev);
  p->tc = T_k_dev != nullptr && in_dtype == WUSHKV_BF16 && n1 - ta >= TC_MIN_TOKENS &&
          (kv_addr & 15) == 0 && (int64_t)batch * n_tok < 2147483647LL &&
          (c.quantizer == WUSHKV_QUEST_INT || (c.clip_lo_rank <= 2 && c.clip_hi_rank >= 127));
  const int64_t tc_qa = p->tc ? ta / 4 : 0;
  // the FMA kernel takes every quad before the tensor-core range
  auto add = [&](int64_t qa, int64_t qb) {
    if (p->tc && qb > tc_qa) qb = tc_qa;
    if (qb <= qa) return;
    p->range[p->nranges][0] = qa;
    p->range[p->nranges][1] = qb;
    ++p->nranges;
  };
  // New tokens may reuse ring slots that old flushed tokens are read from
  // only when the touched span exceeds the ring; then flush first.
  if (has_old_flush && (n1 - (S + P0) > W)) {
    const int64_t q_mid = (flush_end + 3) / 4;
    add(q_begin, q_mid);
    add(q_mid, q_end);
  } else {
    add(q_begin, q_end);
  }
  if (p->tc) {
    PrefillArgs& pf = p->pf;
    pf.c = a.c;
    pf.T = T_k_dev;
    pf.n_tok = n_tok;
    pf.n0 = n0;
    pf.ta = (int)ta;
    pf.tb = (int)n1;
    pf.packed1 = (int)P1;
    pf.tiles_per_unit = (int)((n1 - ta + 127) / 128);
    const int64_t head_tiles = (int64_t)batch * pf.tiles_per_unit;
    // one CTA per SM shared among the heads, each CTA at least
    // TC_MIN_CTA_TILES tiles (the T split into smem is paid once per CTA)
    int64_t per_head = device_sms() / c.n_kv_heads;
    const int64_t by_work = (head_tiles + TC_MIN_CTA_TILES - 1) / TC_MIN_CTA_TILES;
    if (per_head > by_work) per_head = by_work;
    if (per_head < 1) per_head = 1;
    pf.ctas_per_head = (int)per_head;
  }
}

// The whole-cache plan of a one-call append when every sequence holds the
// same number of tokens; ECAPACITY if it would exceed max_ctx.
wushkv_status plan_append(wushkv_cache* cache, const void* k_rope_dev, const void* v_dev, int32_t in_dtype,
                          const float* T_k_dev, int32_t n_tok, int32_t bits, int32_t quantizer,
                          AppendPlan* p) {
  wushkv_status st = check_append_args(cache, k_rope_dev, v_dev, in_dtype, T_k_dev, bits, quantizer);
  if (st != WUSHKV_OK) return st;
  if (n_tok < 0) return WUSHKV_EINVAL;
  if (cache->n + n_tok > cache->cfg.max_ctx) return WUSHKV_ECAPACITY;
  plan_append_view(cache, dev_view(cache), cache->cfg.batch, cache->n, n_tok, k_rope_dev, v_dev, in_dtype,
                   T_k_dev, p);
  return WUSHKV_OK;
}

cudaError_t run_append(AppendPlan& p, const void* k_rope_dev, const void* v_dev, cudaStream_t s) {
  for (int r = 0; r < p.nranges; ++r) {
    set_quad_range(p.a, p.range[r][0], p.range[r][1]);
    const cudaError_t e = launch_append(p.a, s);
    if (e != cudaSuccess) return e;
  }
  if (p.tc) return launch_prefill_tc(p.pf, k_rope_dev, v_dev, device_sms(), s);
  return cudaSuccess;
}

void set_uniform(wushkv_cache* cache) {
  const auto& v = cache->seq_n;
  cache->uniform = true;
  for (size_t b = 1; b < v.size(); ++b) cache->uniform &= v[b] == v[0];
  cache->n = cache->uniform ? v[0] : -1;
}

// Append n_new[b] tokens to sequence b (token-major input, the sequences'
// tokens one after another), each sequence through its own batch-1 view.
// The caller has checked the arguments and the capacity.
wushkv_status append_per_sequence(wushkv_cache* cache, const void* k_rope_dev, const void* v_dev,
                                  int32_t in_dtype, const float* T_k_dev, const int32_t* n_new,
                                  cudaStream_t s) {
  const wushkv_config& c = cache->cfg;
  const size_t row = (size_t)c.n_kv_heads * D * dtype_bytes(in_dtype);
  size_t off = 0;
  for (int b = 0; b < c.batch; ++b) {
    if (n_new[b] == 0) continue;
    AppendPlan p;
    const uint8_t* kb = static_cast<const uint8_t*>(k_rope_dev) + off * row;
    const uint8_t* vb = static_cast<const uint8_t*>(v_dev) + off * row;
    plan_append_view(cache, seq_view(cache, b), 1, cache->seq_n[b], n_new[b], kb, vb, in_dtype, T_k_dev, &p);
    if (run_append(p, kb, vb, s) != cudaSuccess) return WUSHKV_ECUDA;
    cache->seq_n[b] += n_new[b];
    off += (size_t)n_new[b];
  }
  set_uniform(cache);
  return WUSHKV_OK;
}

wushkv_status check_query_args(const void* q_dev, int32_t q_dtype, const float* T_k_invT_dev,
                               const float* q_out_dev, int32_t batch, int32_t n_q_heads, int32_t n_kv_heads) {
  if (!q_dev || !T_k_invT_dev || !q_out_dev || !valid_dtype(q_dtype)) return WUSHKV_EINVAL;
  if (reinterpret_cast<uintptr_t>(T_k_invT_dev) & 15) return WUSHKV_EINVAL;  // read as float4
  if (batch < 1 || n_kv_heads < 1 || n_q_heads < 1 || n_q_heads % n_kv_heads) return WUSHKV_EINVAL;
  const int g = n_q_heads / n_kv_heads;
  if (g != 1 && g != 2 && g != 4 && g != 8 && g != 16) return WUSHKV_EUNSUPPORTED;
  if ((int64_t)batch * n_kv_heads > 2147483647LL) return WUSHKV_EUNSUPPORTED;
  return WUSHKV_OK;
}

wushkv_status check_decode_args(const float* q_prime_dev, const wushkv_cache* cache, const float* out_dev,
                                float scale) {
  if (!q_prime_dev || !cache || !out_dev) return WUSHKV_EINVAL;
  if ((reinterpret_cast<uintptr_t>(out_dev) | reinterpret_cast<uintptr_t>(q_prime_dev)) & 15)
    return WUSHKV_EINVAL;  // read and written as float4
  if (!(scale >= 0.f) || std::isinf(scale)) return WUSHKV_EINVAL;
  return WUSHKV_OK;
}

}  // namespace

extern "C" {

wushkv_status wushkv_append(wushkv_cache* cache, const void* k_rope_dev, const void* v_dev,
                            int32_t in_dtype, const float* T_k_dev, int32_t n_tok, int32_t bits,
                            int32_t quantizer, void* stream) {
  if (cache && !cache->uniform) {   // sequences of unequal lengths: one plan per sequence
    wushkv_status st = check_append_args(cache, k_rope_dev, v_dev, in_dtype, T_k_dev, bits, quantizer);
    if (st != WUSHKV_OK) return st;
    if (n_tok < 0) return WUSHKV_EINVAL;
    for (int64_t n : cache->seq_n)
      if (n + n_tok > cache->cfg.max_ctx) return WUSHKV_ECAPACITY;
    if (n_tok == 0) return WUSHKV_OK;
    std::vector<int32_t> counts((size_t)cache->cfg.batch, n_tok);
    return append_per_sequence(cache, k_rope_dev, v_dev, in_dtype, T_k_dev, counts.data(),
                               static_cast<cudaStream_t>(stream));
  }
  AppendPlan p;
  const wushkv_status st = plan_append(cache, k_rope_dev, v_dev, in_dtype, T_k_dev, n_tok, bits, quantizer, &p);
  if (st != WUSHKV_OK || n_tok == 0) return st;
  if (run_append(p, k_rope_dev, v_dev, static_cast<cudaStream_t>(stream)) != cudaSuccess) return WUSHKV_ECUDA;
  cache->n = p.n1;
  for (auto& n : cache->seq_n) n = p.n1;
  return WUSHKV_OK;
}

wushkv_status wushkv_append_varlen(wushkv_cache* cache, const void* k_rope_dev, const void* v_dev,
                                   int32_t in_dtype, const float* T_k_dev, const int32_t* n_new_host,
                                   int32_t bits, int32_t quantizer, void* stream) {
  wushkv_status st = check_append_args(cache, k_rope_dev, v_dev, in_dtype, T_k_dev, bits, quantizer);
  if (st != WUSHKV_OK) return st;
  if (!n_new_host) return WUSHKV_EINVAL;
  const wushkv_config& c = cache->cfg;
  bool equal = true;
  for (int b = 0; b < c.batch; ++b) {
    if (n_new_host[b] < 0) return WUSHKV_EINVAL;
    if (cache->seq_n[b] + n_new_host[b] > c.max_ctx) return WUSHKV_ECAPACITY;
    equal &= n_new_host[b] == n_new_host[0];
  }
  // equal counts on equal lengths: the packed input is [batch][n][Hkv][128],
  // one plan for the whole cache
  if (equal && cache->uniform)
    return wushkv_append(cache, k_rope_dev, v_dev, in_dtype, T_k_dev, n_new_host[0], bits, quantizer, stream);
  return append_per_sequence(cache, k_rope_dev, v_dev, in_dtype, T_k_dev, n_new_host,
                             static_cast<cudaStream_t>(stream));
}

wushkv_status wushkv_reset_sequence(wushkv_cache* cache, int32_t seq) {
  if (!cache || seq < 0 || seq >= cache->cfg.batch) return WUSHKV_EINVAL;
  cache->seq_n[seq] = 0;
  set_uniform(cache);
  return WUSHKV_OK;
}

wushkv_status wushkv_set_page_table(wushkv_cache* cache, const int32_t* page_table_dev, int32_t max_pages_per_seq) {
  if (!cache || cache->cfg.num_pages <= 0 || !page_table_dev) return WUSHKV_EINVAL;
  if (max_pages_per_seq < cache->lay.packed_capacity / 64) return WUSHKV_EINVAL;
  cache->page_table = page_table_dev;
  cache->pt_stride = max_pages_per_seq;
  return WUSHKV_OK;
}

wushkv_status wushkv_decode_step(wushkv_cache* cache, const void* k_rope_dev, const void* v_dev,
                                 int32_t in_dtype, const float* T_k_dev, const void* q_dev, int32_t q_dtype,
                                 const float* T_k_invT_dev, float* q_prime_dev, float* out_dev, float scale,
                                 void* stream) {
  if (!cache) return WUSHKV_EINVAL;
  const wushkv_config& c = cache->cfg;
  wushkv_status st = check_query_args(q_dev, q_dtype, T_k_invT_dev, q_prime_dev, c.batch, c.n_q_heads,
                                      c.n_kv_heads);
  if (st != WUSHKV_OK) return st;
  st = check_decode_args(q_prime_dev, cache, out_dev, scale);
  if (st != WUSHKV_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const RaggedTable* rt = nullptr;
  DecodeArgs a;
  if (!cache->uniform) {   // sequences of unequal lengths: per-sequence appends, then the query transform
    st = wushkv_append(cache, k_rope_dev, v_dev, in_dtype, T_k_dev, 1, c.bits, c.quantizer, stream);
    if (st != WUSHKV_OK) return st;
    if (launch_query_transform(q_dev, q_dtype, T_k_invT_dev, q_prime_dev, c.batch, c.n_q_heads, c.n_kv_heads,
                               s) != cudaSuccess)
      return WUSHKV_ECUDA;
    st = plan_decode(cache, q_prime_dev, out_dev, scale, &a, &rt);
    if (st != WUSHKV_OK) return st;
    return cuda_status(launch_decode(a, cache->wmaps, rt, s));
  }
  AppendPlan p;
  st = plan_append(cache, k_rope_dev, v_dev, in_dtype, T_k_dev, 1, c.bits, c.quantizer, &p);
  if (st != WUSHKV_OK) return st;
  cudaError_t e;
  const int64_t S = c.sink;
  const bool new_in_window = p.n1 - 1 < S || p.n1 - 1 >= S + p.a.packed1;
  if (!p.tc && p.nranges == 1 && new_in_window) {
    // one launch: the new key's rows, the query rows and the flushed chunk
    const int64_t f0 = (S + p.a.packed0) / 4, f1 = (S + p.a.packed1) / 4;   // quad-aligned
    AppendArgs fa = p.a;
    fa.quad_begin = f0;
    fa.n_quads = f1 - f0;
    fa.quads_per_cta = 1;
    e = launch_step_rows(fa, (int)(f1 - f0), q_dev, q_dtype, T_k_invT_dev, q_prime_dev, s);
  } else if (!p.tc && p.nranges == 1) {   // one launch for the append and the query transform
    set_quad_range(p.a, p.range[0][0], p.range[0][1]);
    e = launch_append_qt(p.a, q_dev, q_dtype, T_k_invT_dev, q_prime_dev, s);
  } else {
    e = run_append(p, k_rope_dev, v_dev, s);
    if (e == cudaSuccess)
      e = launch_query_transform(q_dev, q_dtype, T_k_invT_dev, q_prime_dev, c.batch, c.n_q_heads,
                                 c.n_kv_heads, s);
  }
  if (e != cudaSuccess) return WUSHKV_ECUDA;
  cache->n = p.n1;
  for (auto& n : cache->seq_n) n = p.n1;
  st = plan_decode(cache, q_prime_dev, out_dev, scale, &a, &rt);
  if (st != WUSHKV_OK) return st;
  return cuda_status(launch_decode(a, cache->wmaps, rt, s));
}

wushkv_status wushkv_prefill_attention(const float* q_prime_dev, const wushkv_cache* cache, float* out_dev,
                                       int32_t n_q, float scale, void* stream) {
  wushkv_status st = check_decode_args(q_prime_dev, cache, out_dev, scale);
  if (st != WUSHKV_OK) return st;
  const wushkv_config& c = cache->cfg;
  if (!cache->uniform) return WUSHKV_EUNSUPPORTED;   // one count for every sequence
  if (n_q < 1 || n_q > cache->n) return WUSHKV_EINVAL;
  if (c.num_pages > 0 && cache->page_table == nullptr) return WUSHKV_EINVAL;
  const int64_t units = (int64_t)c.batch * c.n_kv_heads;
  if (units > 65535) return WUSHKV_EUNSUPPORTED;   // one grid row per unit
  PaArgs a;
  std::memset(&a, 0, sizeof(a));
  a.c = dev_view(cache);
  a.q = q_prime_dev;
  a.out = out_dev;
  a.n = (int)cache->n;
  a.n_q = n_q;
  a.ns = (int)std::min<int64_t>(cache->n, c.sink);
  a.P = (int)packed_count(cache->n, c);
  const float sc = scale > 0.f ? scale : 0.08838834764831845f;  // 1/sqrt(128)
  a.scale_log2 = sc * 1.4426950408889634f;
  return cuda_status(launch_prefill_attention(a, static_cast<cudaStream_t>(stream)));
}

wushkv_status wushkv_query_transform(const void* q_dev, int32_t q_dtype, const float* T_k_invT_dev,
                                     float* q_out_dev, int32_t batch, int32_t n_q_heads,
                                     int32_t n_kv_heads, void* stream) {
  const wushkv_status st = check_query_args(q_dev, q_dtype, T_k_invT_dev, q_out_dev, batch, n_q_heads, n_kv_heads);
  if (st != WUSHKV_OK) return st;
  return cuda_status(launch_query_transform(q_dev, q_dtype, T_k_invT_dev, q_out_dev, batch,
                                            n_q_heads, n_kv_heads, static_cast<cudaStream_t>(stream)));
}

wushkv_status wushkv_decode(const float* q_prime_dev, const wushkv_cache* cache, float* out_dev,
                            float scale, void* stream) {
  wushkv_status st = check_decode_args(q_prime_dev, cache, out_dev, scale);
  if (st != WUSHKV_OK) return st;
  DecodeArgs a;
  const RaggedTable* rt = nullptr;
  st = plan_decode(cache, q_prime_dev, out_dev, scale, &a, &rt);
  if (st != WUSHKV_OK) return st;
  return cuda_status(launch_decode(a, cache->wmaps, rt, static_cast<cudaStream_t>(stream)));
}

wushkv_status wushkv_export(const wushkv_cache* cache, int32_t seq, int32_t head, int32_t kv,
                            int32_t tok0, int32_t ntok, uint8_t* codes_host, uint16_t* meta_host,
                            uint16_t* fp16_host, int8_t* kinds_host) {
  if (!cache) return WUSHKV_EINVAL;
  const wushkv_config& c = cache->cfg;
  const wushkv_layout& L = cache->lay;
  if (seq < 0 || seq >= c.batch || head < 0 || head >= c.n_kv_heads || (kv != 0 && kv != 1))
    return WUSHKV_EINVAL;
  const int64_t n = cache->seq_n[seq];
  if (tok0 < 0 || ntok < 0 || (int64_t)tok0 + ntok > n) return WUSHKV_EINVAL;
  const size_t u = (size_t)seq * c.n_kv_heads + head;
  const int64_t ns = n < c.sink ? n : c.sink;
  const int64_t P = packed_count(n, c);
  const int W = L.ring_slots;
  // copy the unit's block records (they hold K and V) to host, one after
  // another; a paged cache's through the sequence's page-table row
  const int64_t nblk = (P + 63) / 64;
  std::vector<uint8_t> packed((size_t)(nblk > 0 ? nblk : 1) * L.block_stride);
  if (c.num_pages > 0 && nblk > 0) {
    if (!cache->page_table) return WUSHKV_EINVAL;
    std::vector<int32_t> pages((size_t)nblk);
    if (cudaMemcpy(pages.data(), cache->page_table + (size_t)seq * cache->pt_stride, nblk * sizeof(int32_t),
                   cudaMemcpyDeviceToHost))
      return WUSHKV_ECUDA;
    for (int64_t i = 0; i < nblk; ++i) {
      if (pages[i] < 0 || pages[i] >= c.num_pages) return WUSHKV_EINVAL;
      if (cudaMemcpy(packed.data() + i * L.block_stride,
                     cache->base + ((size_t)pages[i] * c.n_kv_heads + head) * L.block_stride, L.block_stride,
                     cudaMemcpyDeviceToHost))
        return WUSHKV_ECUDA;
    }
  } else if (nblk > 0 &&
             cudaMemcpy(packed.data(), cache->base + u * L.unit_stride, nblk * L.block_stride,
                        cudaMemcpyDeviceToHost)) {
    return WUSHKV_ECUDA;
  }
  auto word_at = [&](uint64_t part_off, int64_t blk, size_t byte) {
    uint32_t wd;
    std::memcpy(&wd, packed.data() + (size_t)blk * L.block_stride + part_off + byte, 4);
    return wd;
  };
  std::vector<uint16_t> sink((size_t)c.sink * 128), ring((size_t)W * 128);
  if (c.sink > 0 &&
      cudaMemcpy(sink.data(), cache->base + (kv == 0 ? L.sink_k_off : L.sink_v_off) + u * L.sink_unit_stride,
                 L.sink_unit_stride, cudaMemcpyDeviceToHost))
    return WUSHKV_ECUDA;
  if (cudaMemcpy(ring.data(), cache->base + (kv == 0 ? L.ring_k_off : L.ring_v_off) + u * L.ring_unit_stride,
                 L.ring_unit_stride, cudaMemcpyDeviceToHost))
    return WUSHKV_ECUDA;
  const int mb = (int)L.meta_bytes / 2;
  for (int i = 0; i < ntok; ++i) {
    const int64_t t = tok0 + i;
    int kind;
    if (t < ns) kind = 0;
    else if (t < ns + P) kind = 1;
    else kind = 2;
    if (kinds_host) kinds_host[i] = (int8_t)kind;
    if (kind == 1) {
      const int64_t pk = t - c.sink;
      uint8_t code[128] = {0};
      int shift = 0;
      for (int p = 0; p < L.n_planes; ++p) {
        const int w = L.plane_bits[p], F = 8 / w;
        const uint32_t mask = (1u << w) - 1u;
        for (int d = 0; d < 128; ++d) {
          uint32_t wd;
          int bit;
          if (kv == 0 && c.bits == 2) {   // K quads
            const int64_t quad = pk / 4;
            wd = word_at(L.k_plane_off[p], quad / 16,
                         (size_t)(quad % 16) * 128 + 4 * (size_t)k2_word_pos(quad, d / 4));
            bit = 8 * (d % 4) + 2 * (int)(pk % 4);
          } else if (kv == 0) {
            const int ks = d / 32, rem = d % 32, h2 = rem / 16, c4 = (rem % 16) / 4, beta = d % 4;
            const int rho = 4 * h2 + ks;
            wd = word_at(L.k_plane_off[p], pk / 64, (size_t)k_row_pos(pk) * 16 * w + 4 * (c4 * w + rho / F));
            bit = 8 * beta + w * (rho % F);
          } else {
            const int mt = d / 16, rem = d % 16, rh = rem / 8, r = rem % 8;
            const int rho = 2 * mt + rh, beta = (int)(pk % 4);
            const int quad = (int)(pk / 4);
            wd = word_at(L.v_plane_off[p], quad / 16,
                         (size_t)(quad % 16) * 64 * w + 4 * v_word_index(quad, r, rho / F, w));
            bit = 8 * beta + w * (rho % F);
          }
          code[d] |= (uint8_t)(((wd >> bit) & mask) << shift);
        }
        shift += w;
      }
      if (codes_host) std::memcpy(codes_host + (size_t)i * 128, code, 128);
      if (meta_host) {
        const uint8_t* m = packed.data() + (size_t)(pk / 64) * L.block_stride +
                           (kv == 0 ? L.k_meta_off : L.v_meta_off) + (size_t)(pk % 64) * L.meta_bytes;
        std::memcpy(&meta_host[2 * i], m, 2);
        if (mb == 2) std::memcpy(&meta_host[2 * i + 1], m + 2, 2);
        else meta_host[2 * i + 1] = 0;
      }
      if (fp16_host) std::memset(fp16_host + (size_t)i * 128, 0, 256);
    } else {
      const uint16_t* row = kind == 0 ? &sink[(size_t)t * 128]
                                      : &ring[(size_t)((t - c.sink) % W) * 128];
      if (fp16_host) std::memcpy(fp16_host + (size_t)i * 128, row, 256);
      if (codes_host) std::memset(codes_host + (size_t)i * 128, 0, 128);
      if (meta_host) { meta_host[2 * i] = 0; meta_host[2 * i + 1] = 0; }
    }
  }
  return WUSHKV_OK;
}

void wushkv_inject_decode_timeout(uint32_t polls) { g_inject_polls.store(polls, std::memory_order_relaxed); }

wushkv_status wushkv_device_status(const wushkv_cache* cache, int32_t clear, int32_t* out) {
  if (!cache || !out) return WUSHKV_EINVAL;
  int32_t v = 0;
  if (cudaMemcpy(&v, cache->base + cache->lay.status_off, 4, cudaMemcpyDeviceToHost))
    return WUSHKV_ECUDA;
  if (clear && cudaMemset(cache->base + cache->lay.status_off, 0, 4)) return WUSHKV_ECUDA;
  *out = v;
  return WUSHKV_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at decode time: code running inside a
// host allocator hook, plug-ins whose host application owns every device
// allocation, or engines that forbid allocation after start-up.  For them
// the split-K partials and arrival counters of the decode live in this
// file-scope device array instead of the cache buffer's workspace.  The
// array is a fixed 8 MiB and stays resident on every GPU that loads the
// library until the process exits.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t NOALLOC_SCRATCH_BYTES = size_t(8) << 20;
constexpr size_t NOALLOC_COUNTER_BYTES = size_t(65536) * sizeof(int);  // one per unit

static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch, looked up once per device (by
// whichever thread gets there first; the lookup is idempotent).  In host
// code the symbol itself is only a host-side stand-in for the array.
std::atomic<void*> g_noalloc_addr[64];

}  // namespace

extern "C" wushkv_status wushkv_decode_noalloc(const float* q_prime_dev, const wushkv_cache* cache,
                                                float* out_dev, float scale, void* stream) {
  if (!q_prime_dev || !cache || !out_dev) return WUSHKV_EINVAL;
  if ((reinterpret_cast<uintptr_t>(out_dev) | reinterpret_cast<uintptr_t>(q_prime_dev)) & 15)
    return WUSHKV_EINVAL;  // read and written as float4
  if (!(scale >= 0.f) || std::isinf(scale)) return WUSHKV_EINVAL;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return WUSHKV_ECUDA;
  if (dev < 0 || dev >= 64) return WUSHKV_EUNSUPPORTED;
  void* scratch = g_noalloc_addr[dev].load(std::memory_order_acquire);
  if (!scratch) {
    if (cudaGetSymbolAddress(&scratch, g_noalloc_scratch) != cudaSuccess || !scratch) return WUSHKV_ECUDA;
    g_noalloc_addr[dev].store(scratch, std::memory_order_release);
  }
  DecodeArgs a;
  const RaggedTable* rt = nullptr;
  const wushkv_status st = plan_decode(cache, q_prime_dev, out_dev, scale, &a, &rt);
  if (st != WUSHKV_OK) return st;
  // Partials are packed densely, as many per unit as CTAs of this call can
  // touch one unit.
  const int64_t items = (int64_t)a.cta_q * a.grid + a.cta_r;
  int64_t ni_max = a.items_per_unit;
  if (rt)
    for (int b = 0; b < rt->nseq; ++b)
      ni_max = std::max<int64_t>(ni_max, (rt->item_start[b + 1] - rt->item_start[b]) / cache->cfg.n_kv_heads);
  const int total = (int)parts_per_unit_bound(items, a.grid, ni_max);
  a.c.max_splits = total;
  const size_t units = (size_t)a.c.units;
  const size_t partial_bytes = units * (size_t)total * a.c.group * PARTIAL_FLOATS * sizeof(float);
  if (units * sizeof(int) > NOALLOC_COUNTER_BYTES ||
      partial_bytes > NOALLOC_SCRATCH_BYTES - NOALLOC_COUNTER_BYTES)
    return WUSHKV_ECAPACITY;
  unsigned char* base = static_cast<unsigned char*>(scratch);
  a.counters = reinterpret_cast<int*>(base);
  a.partials = reinterpret_cast<float*>(base + NOALLOC_COUNTER_BYTES);
  a.c.counters = a.counters;
  a.c.counter_stride = 1;
  a.c.partials = a.partials;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The array keeps the previous call's contents: arrival counters must
  // start at zero.
  if (cudaMemsetAsync(a.counters, 0, units * sizeof(int), s) != cudaSuccess) return WUSHKV_ECUDA;
  return cuda_status(launch_decode(a, cache->wmaps, rt, s));
}
