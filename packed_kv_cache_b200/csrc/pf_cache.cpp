// pf_cache.cpp -- host side of the packed KV cache: argument checks, the
// per-layer partition state machine, arena layout, tensor-map encoding and
// kernel launches.  Implements the C ABI declared in include/pf.h.
//
// Partitions and their update rules follow PackForcing (arXiv): "Sink
// Tokens" (first blocks, never evicted), "Compressed Mid Tokens" (a pool of
// compressed blocks), "Recent & Current Tokens", "Dual-Resolution Shifting
// Mechanism" (a block's compressed copy is computed with it and joins the
// pool when the block leaves the recent partition) and "The Position
// Misalignment Problem" (the oldest compressed block is evicted when the
// pool is full).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "pf.h"
#include "pf_internal.h"

namespace {

thread_local std::string g_last_error;

pf_status fail(pf_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

pf_status cuda_fail(cudaError_t e, const char* what) {
  return fail(PF_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

constexpr size_t kAlign = 256;
constexpr long long kDefaultTimeoutCycles = 4000000000LL;  // about 2 s at 2 GHz
constexpr int kMaxPoolSlots = 8192;                         // the top-k keeps all scores in shared memory

// attention scratch shared by all layers: split-tail partial outputs, row
// statistics and tickets
constexpr size_t kAttendScratchBytes = pf::kAttendPartOBytes + pf::kAttendPartMLBytes;

struct Geometry {
  int n, n_c, slots, HD;
  size_t sink_bytes, pool_bytes, recent_bytes;  // per K (or V) tensor
  size_t sel_bytes, scores_bytes, partial_bytes, qsum_bytes, ticket_bytes, kbar_bytes;
  size_t layer_bytes, arena_bytes;
  int chunk_rows, chunks_per_block;
};

pf_status check_config(const pf_config* c) {
  if (c == nullptr) return fail(PF_ERR_ARG, "config is NULL");
  if (c->layers <= 0 || c->batch <= 0 || c->heads <= 0 || c->block_frames <= 0 || c->h <= 0 || c->w <= 0)
    return fail(PF_ERR_ARG, "layers, batch, heads, block_frames, h and w must be positive");
  if (c->head_dim != pf::kHeadDim) return fail(PF_ERR_UNSUPPORTED, "head_dim must be 128 (got %d)", c->head_dim);
  if (c->sink_blocks < 0 || c->recent_blocks < 1 || c->mid_capacity < 0 || c->n_top < 0)
    return fail(PF_ERR_ARG, "need sink_blocks >= 0, recent_blocks >= 1, mid_capacity >= 0, n_top >= 0");
  const int* s = c->rope_split;
  if (s[0] < 0 || s[1] < 0 || s[2] < 0 || (s[0] & 1) || (s[1] & 1) || (s[2] & 1) ||
      s[0] + s[1] + s[2] != c->head_dim)
    return fail(PF_ERR_UNSUPPORTED, "rope_split must be three even sizes summing to head_dim");
  if (s[0] > 64) return fail(PF_ERR_UNSUPPORTED, "at most 64 temporal rotary dims (got %d)", s[0]);
  if (!(c->rope_base > 1.0f)) return fail(PF_ERR_ARG, "rope_base must be > 1");
  if (c->sink_rope_in_attention != 0 && c->sink_rope_in_attention != 1)
    return fail(PF_ERR_ARG, "sink_rope_in_attention must be 0 or 1");
  long long n = 1LL * c->block_frames * c->h;  // both positive ints: no overflow
  if (n <= (1 << 24)) n *= c->w;                 // nor here
  if (n > (1 << 24)) return fail(PF_ERR_CAPACITY, "a block holds at most 2^24 tokens (B_f * h * w)");
  const long long n_c = 1LL * (c->block_frames / 2) * (c->h / 4) * (c->w / 4);
  if (n_c <= 0 && c->mid_capacity > 0)
    return fail(PF_ERR_ARG, "compressed blocks would be empty (B_f >= 2, h >= 4, w >= 4 needed)");
  if (1LL * c->mid_capacity + c->recent_blocks > kMaxPoolSlots)
    return fail(PF_ERR_CAPACITY, "mid_capacity + recent_blocks must be <= %d", kMaxPoolSlots);
  // the scoring kernel keeps the pooled query (H * D floats) and every pool
  // score (kMaxPoolSlots keys) in shared memory: 128 KB + 32 KB at most
  if (1LL * c->heads * c->head_dim > 32768) return fail(PF_ERR_CAPACITY, "H * D must be <= 32768 (at most 256 heads)");
  // The attention kernel walks the context in 32-key sub-boxes, counted in
  // int, and finds a sub-box's block by a float-reciprocal quotient that is
  // exact below 2^22 sub-boxes: the context, padded as the kernel pads it,
  // stays below 2^27 keys.
  const long long sub = 32;
  const long long blk_keys = (n + sub - 1) / sub * sub;
  const long long mid_keys = n_c > 0 ? (n_c + sub - 1) / sub * sub * std::min(c->n_top, c->mid_capacity) : 0;
  const long long sink_keys = (c->sink_blocks * n + sub - 1) / sub * sub;
  const long long context = sink_keys + mid_keys + (c->recent_blocks + 1LL) * blk_keys;
  if (context >= (1LL << 27))
    return fail(PF_ERR_CAPACITY, "attention context of %lld keys (in 32-key sub-boxes) must stay below 2^27",
                context);
  return PF_OK;
}

// Size arithmetic that records an overflow instead of wrapping around: a
// wrapped arena size would let the partitions of a huge configuration be
// laid out past the end of the caller's arena.
struct Sizes {
  bool overflow = false;
  size_t mul(size_t a, size_t b) {
    size_t r = 0;
    if (__builtin_mul_overflow(a, b, &r)) overflow = true;
    return r;
  }
  size_t add(size_t a, size_t b) {
    size_t r = 0;
    if (__builtin_add_overflow(a, b, &r)) overflow = true;
    return r;
  }
  size_t aligned(size_t x) { return mul(add(x, kAlign - 1) / kAlign, kAlign); }
  size_t bytes(size_t a, size_t b, size_t c, size_t d = 1) { return aligned(mul(mul(a, b), mul(c, d))); }
};

// Sets *overflow when a size does not fit in size_t.
Geometry geometry(const pf_config* c, bool* overflow) {
  Geometry g;
  Sizes z;
  g.n = c->block_frames * c->h * c->w;
  g.n_c = (c->block_frames / 2) * (c->h / 4) * (c->w / 4);
  if (g.n_c < 1) g.n_c = 1;  // pool unused (mid_capacity == 0); keep the maps well formed
  g.slots = c->mid_capacity + c->recent_blocks;
  g.HD = c->heads * c->head_dim;
  const size_t row = static_cast<size_t>(g.HD) * 2;
  const size_t B = static_cast<size_t>(c->batch);
  g.sink_bytes = z.bytes(B, c->sink_blocks, g.n, row);
  g.pool_bytes = z.bytes(B, g.slots, g.n_c, row);
  g.recent_bytes = z.bytes(B, c->recent_blocks, g.n, row);
  g.chunk_rows = 32;
  g.chunks_per_block = (g.n_c + g.chunk_rows - 1) / g.chunk_rows;
  // selection scratch: per-row-chunk query sums, per-slab partial scores of
  // every slot, and the batch and slab tickets
  const int slabs = g.HD / pf::kSelSlabCols;
  g.sel_bytes = z.bytes(B, c->n_top > 0 ? c->n_top : 1, 4);
  g.scores_bytes = z.bytes(B, g.slots, 4);
  g.partial_bytes = z.bytes(B, g.slots, g.chunks_per_block, 4);
  // per-row-chunk query sums, then their total
  g.qsum_bytes = z.bytes(B, pf::kSelMaxRowChunks + 1, g.HD, 4);
  g.ticket_bytes = z.bytes(B, 1 + slabs, 4);
  g.kbar_bytes = z.bytes(B, g.slots, g.HD, 4);
  size_t t = z.mul(2, z.add(z.add(g.sink_bytes, g.pool_bytes), g.recent_bytes));
  t = z.add(t, z.add(z.add(g.sel_bytes, g.scores_bytes), g.partial_bytes));
  t = z.add(t, z.add(z.add(g.qsum_bytes, g.ticket_bytes), g.kbar_bytes));
  g.layer_bytes = t;
  g.arena_bytes = z.add(kAlign /* error word */ + kAttendScratchBytes, z.mul(g.layer_bytes, c->layers));
  *overflow = z.overflow;
  return g;
}

struct Layer {
  int blocks_seen = 0, sink_filled = 0;
  int recent_count = 0, recent_head = 0;
  int mid_count = 0, mid_head = 0;
  bool sel_valid = false;
  int n_sel = 0;
  long long evicted = 0, total_shift = 0;
  char *sink_k, *sink_v, *pool_k, *pool_v, *recent_k, *recent_v;
  int32_t* sel;
  float *scores, *partial, *qsum;
  unsigned* ticket;       // [B] batch tickets, then [B, H * D / 64] slab tickets
  float* kbar;  // [B, slots, H * D] mean key of each pool slot
  // the attention's tensor maps over this layer's partitions (sink, mid
  // pool, recent ring), encoded at the layer's first pf_attend: the arena
  // does not move, so they stay valid for the cache's life
  bool maps_ready = false;
  CUtensorMap tm_k[3], tm_v[3];
};

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn lookup_encode_fn() {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    return reinterpret_cast<EncodeTiledFn>(p);
  return nullptr;
}

// looked up once per process (thread-safe initialisation of a local static)
EncodeTiledFn get_encode_fn() {
  static const EncodeTiledFn fn = lookup_encode_fn();
  return fn;
}

}  // namespace

namespace pf {
CUresult encode_tiled(CUtensorMap* m, CUtensorMapDataType dtype, int rank, void* base, const cuuint64_t* dims,
                      const cuuint64_t* strides, const cuuint32_t* box, CUtensorMapSwizzle swizzle,
                      CUtensorMapL2promotion l2) {
  EncodeTiledFn fn = get_encode_fn();
  if (fn == nullptr) return CUDA_ERROR_NOT_SUPPORTED;
  const cuuint32_t estr[5] = {1u, 1u, 1u, 1u, 1u};
  return fn(m, dtype, static_cast<cuuint32_t>(rank), base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            swizzle, l2, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

int report_error(int status, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return status;
}
}  // namespace pf

struct pf_cache {
  pf_config cfg;
  Geometry g;
  char* arena;
  size_t arena_bytes;
  unsigned* err;  // device error word
  float* part_o;
  float* part_ml;
  long long timeout_cycles;
  std::vector<Layer> L;
};

namespace {

pf_status check_layer(const pf_cache* c, int layer) {
  if (c == nullptr) return fail(PF_ERR_ARG, "cache is NULL");
  if (layer < 0 || layer >= c->cfg.layers) return fail(PF_ERR_ARG, "layer %d out of range [0, %d)", layer, c->cfg.layers);
  return PF_OK;
}

pf_status check_ptr(const void* p, const char* name) {
  if (p == nullptr) return fail(PF_ERR_ARG, "%s is NULL", name);
  if (reinterpret_cast<uintptr_t>(p) % 16 != 0) return fail(PF_ERR_ARG, "%s is not 16-byte aligned", name);
  return PF_OK;
}

// 4-D map (D, H, rows, segs) over a bf16 [segs, rows, H, D] tensor with
// 64-dim x `box_rows` boxes and 128-byte swizzle.
pf_status encode_map(CUtensorMap* m, const void* base, int H, long long rows, long long segs, int box_rows) {
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(pf::kHeadDim), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(segs)};
  const cuuint64_t rowb = static_cast<cuuint64_t>(pf::kHeadDim) * 2;
  const cuuint64_t strides[3] = {rowb, rowb * H, rowb * H * static_cast<cuuint64_t>(rows)};
  const cuuint32_t box[4] = {64u, 1u, static_cast<cuuint32_t>(box_rows), 1u};
  const CUresult r = pf::encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
                                      box, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
  if (r == CUDA_ERROR_NOT_SUPPORTED) return fail(PF_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable (driver too old?)");
  if (r != CUDA_SUCCESS) return fail(PF_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return PF_OK;
}

struct RunBuilder {
  pf::RowRuns runs;
  pf::RopeTable tab;
  cudaStream_t st;
  bool f32 = false;  // runs of float32 vectors (cached mean keys) instead of bf16 keys
  cudaError_t err = cudaSuccess;
  RunBuilder() { runs.n = 0; runs.start[0] = 0; }
  void flush() {
    if (runs.n == 0) return;
    cudaError_t e = f32 ? pf::launch_rope_shift_f32(runs, tab, st) : pf::launch_rope_shift(runs, tab, st);
    if (e != cudaSuccess && err == cudaSuccess) err = e;
    runs.n = 0;
    runs.start[0] = 0;
  }
  void add(void* ptr, long long row_heads) {
    if (row_heads <= 0) return;
    if (runs.n == pf::kMaxSegs) flush();
    runs.ptr[runs.n] = ptr;
    runs.start[runs.n + 1] = runs.start[runs.n] + row_heads;
    ++runs.n;
  }
};

struct CopyBuilder {
  pf::CopyRuns runs;
  cudaStream_t st;
  cudaError_t err = cudaSuccess;
  CopyBuilder() { runs.n = 0; runs.start[0] = 0; }
  void flush() {
    if (runs.n == 0) return;
    cudaError_t e = pf::launch_copy(runs, st);
    if (e != cudaSuccess && err == cudaSuccess) err = e;
    runs.n = 0;
    runs.start[0] = 0;
  }
  void add(void* dst, const void* src, size_t bytes) {
    if (bytes == 0) return;
    if (runs.n == pf::kMaxSegs) flush();
    runs.dst[runs.n] = dst;
    runs.src[runs.n] = src;
    runs.start[runs.n + 1] = runs.start[runs.n] + static_cast<long long>(bytes / 16);
    ++runs.n;
  }
};

int context_tokens(const pf_cache* c, const Layer& Ly) {
  const int n_sel = (c->cfg.n_top >= Ly.mid_count) ? Ly.mid_count : (Ly.sel_valid ? Ly.n_sel : c->cfg.n_top);
  return Ly.sink_filled * c->g.n + n_sel * c->g.n_c + Ly.recent_count * c->g.n + c->g.n;
}

}  // namespace

extern "C" {

int pf_version(void) { return 100; }

const char* pf_last_error(void) { return g_last_error.c_str(); }

const char* pf_status_string(pf_status s) {
  switch (s) {
    case PF_OK: return "PF_OK";
    case PF_ERR_ARG: return "PF_ERR_ARG";
    case PF_ERR_ARENA: return "PF_ERR_ARENA";
    case PF_ERR_STATE: return "PF_ERR_STATE";
    case PF_ERR_CAPACITY: return "PF_ERR_CAPACITY";
    case PF_ERR_CUDA: return "PF_ERR_CUDA";
    case PF_ERR_TIMEOUT: return "PF_ERR_TIMEOUT";
    case PF_ERR_UNSUPPORTED: return "PF_ERR_UNSUPPORTED";
  }
  return "unknown status";
}

pf_status pf_cache_bytes(const pf_config* cfg, size_t* bytes) {
  pf_status s = check_config(cfg);
  if (s != PF_OK) return s;
  if (bytes == nullptr) return fail(PF_ERR_ARG, "bytes is NULL");
  bool overflow = false;
  const Geometry g = geometry(cfg, &overflow);
  if (overflow) return fail(PF_ERR_CAPACITY, "the cache's size does not fit in size_t");
  *bytes = g.arena_bytes;
  return PF_OK;
}

pf_status pf_cache_create(const pf_config* cfg, void* dev_arena, size_t arena_bytes, void* stream, pf_cache** out) {
  size_t need = 0;
  pf_status s = pf_cache_bytes(cfg, &need);
  if (s != PF_OK) return s;
  if (out == nullptr) return fail(PF_ERR_ARG, "out is NULL");
  if (dev_arena == nullptr) return fail(PF_ERR_ARG, "arena is NULL");
  if (reinterpret_cast<uintptr_t>(dev_arena) % kAlign != 0) return fail(PF_ERR_ARENA, "arena is not 256-byte aligned");
  if (arena_bytes < need) return fail(PF_ERR_ARENA, "arena has %zu bytes, %zu needed", arena_bytes, need);
  pf_cache* c = new (std::nothrow) pf_cache();
  if (c == nullptr) return fail(PF_ERR_CAPACITY, "out of host memory");
  c->cfg = *cfg;
  bool overflow = false;
  c->g = geometry(cfg, &overflow);  // no overflow: pf_cache_bytes succeeded
  c->arena = static_cast<char*>(dev_arena);
  c->arena_bytes = arena_bytes;
  c->err = reinterpret_cast<unsigned*>(c->arena);
  c->timeout_cycles = kDefaultTimeoutCycles;
  try {
    c->L.resize(cfg->layers);
  } catch (...) {  // no exception may cross the C ABI
    delete c;
    return fail(PF_ERR_CAPACITY, "out of host memory for %d layers", cfg->layers);
  }
  char* p = c->arena + kAlign;
  c->part_o = reinterpret_cast<float*>(p); p += pf::kAttendPartOBytes;
  c->part_ml = reinterpret_cast<float*>(p); p += pf::kAttendPartMLBytes;
  for (int l = 0; l < cfg->layers; ++l) {
    Layer& Ly = c->L[l];
    const Geometry& g = c->g;
    Ly.sink_k = p; p += g.sink_bytes;
    Ly.sink_v = p; p += g.sink_bytes;
    Ly.pool_k = p; p += g.pool_bytes;
    Ly.pool_v = p; p += g.pool_bytes;
    Ly.recent_k = p; p += g.recent_bytes;
    Ly.recent_v = p; p += g.recent_bytes;
    Ly.sel = reinterpret_cast<int32_t*>(p); p += g.sel_bytes;
    Ly.scores = reinterpret_cast<float*>(p); p += g.scores_bytes;
    Ly.partial = reinterpret_cast<float*>(p); p += g.partial_bytes;
    Ly.qsum = reinterpret_cast<float*>(p); p += g.qsum_bytes;
    Ly.ticket = reinterpret_cast<unsigned*>(p); p += g.ticket_bytes;
    Ly.kbar = reinterpret_cast<float*>(p); p += g.kbar_bytes;
  }
  cudaError_t e = cudaMemsetAsync(c->arena, 0, need, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    delete c;
    return cuda_fail(e, "cudaMemsetAsync(arena)");
  }
  *out = c;
  return PF_OK;
}

pf_status pf_cache_destroy(pf_cache* cache) {
  if (cache == nullptr) return fail(PF_ERR_ARG, "cache is NULL");
  delete cache;
  return PF_OK;
}

pf_status pf_cache_layer_info(const pf_cache* c, int layer, pf_layer_info* out) {
  pf_status s = check_layer(c, layer);
  if (s != PF_OK) return s;
  if (out == nullptr) return fail(PF_ERR_ARG, "out is NULL");
  const Layer& Ly = c->L[layer];
  out->blocks_seen = Ly.blocks_seen;
  out->sink_filled = Ly.sink_filled;
  out->recent_count = Ly.recent_count;
  out->recent_head = Ly.recent_head;
  out->mid_count = Ly.mid_count;
  out->mid_head = Ly.mid_head;
  out->pool_slots = c->g.slots;
  out->selection_valid = Ly.sel_valid ? 1 : 0;
  out->n_selected = (c->cfg.n_top >= Ly.mid_count) ? Ly.mid_count : (Ly.sel_valid ? Ly.n_sel : 0);
  out->context_tokens = context_tokens(c, Ly);
  out->evicted = Ly.evicted;
  out->total_shift = Ly.total_shift;
  out->sink_k = Ly.sink_k;
  out->sink_v = Ly.sink_v;
  out->pool_k = Ly.pool_k;
  out->pool_v = Ly.pool_v;
  out->recent_k = Ly.recent_k;
  out->recent_v = Ly.recent_v;
  out->selection = Ly.sel;
  out->scores = Ly.scores;
  return PF_OK;
}

pf_status pf_cache_append_block(pf_cache* c, int layer, const void* K, const void* V, const void* Kc, const void* Vc,
                                int* evicted, void* stream) {
  pf_status s = check_layer(c, layer);
  if (s != PF_OK) return s;
  if ((s = check_ptr(K, "K")) != PF_OK || (s = check_ptr(V, "V")) != PF_OK) return s;
  Layer& Ly = c->L[layer];
  const pf_config& cf = c->cfg;
  const Geometry& g = c->g;
  const bool to_sink = Ly.sink_filled < cf.sink_blocks;
  if (!to_sink && cf.mid_capacity > 0) {
    if ((s = check_ptr(Kc, "Kc")) != PF_OK || (s = check_ptr(Vc, "Vc")) != PF_OK) return s;
  }
  const size_t row = static_cast<size_t>(g.HD) * 2;
  const size_t blk = static_cast<size_t>(g.n) * row;     // one block, one batch item
  const size_t cblk = static_cast<size_t>(g.n_c) * row;  // one compressed block
  CopyBuilder cb;
  cb.st = static_cast<cudaStream_t>(stream);
  int ev = 0;
  Layer nx = Ly;
  if (to_sink) {
    for (int b = 0; b < cf.batch; ++b) {
      const size_t off = (static_cast<size_t>(b) * cf.sink_blocks + Ly.sink_filled) * blk;
      cb.add(Ly.sink_k + off, static_cast<const char*>(K) + b * blk, blk);
      cb.add(Ly.sink_v + off, static_cast<const char*>(V) + b * blk, blk);
    }
    nx.sink_filled += 1;
  } else {
    if (nx.recent_count == cf.recent_blocks) {
      // the oldest recent block leaves; its compressed copy (already in the
      // pool right after the live blocks) becomes the newest mid block
      nx.recent_head = (nx.recent_head + 1) % cf.recent_blocks;
      nx.recent_count -= 1;
      nx.mid_count += 1;
      if (nx.mid_count > cf.mid_capacity) {
        nx.mid_head = (nx.mid_head + 1) % g.slots;
        nx.mid_count -= 1;
        ev = 1;
      }
      nx.sel_valid = false;
    }
    const int rslot = (nx.recent_head + nx.recent_count) % cf.recent_blocks;
    const int pslot = (nx.mid_head + nx.mid_count + nx.recent_count) % g.slots;
    for (int b = 0; b < cf.batch; ++b) {
      const size_t roff = (static_cast<size_t>(b) * cf.recent_blocks + rslot) * blk;
      cb.add(Ly.recent_k + roff, static_cast<const char*>(K) + b * blk, blk);
      cb.add(Ly.recent_v + roff, static_cast<const char*>(V) + b * blk, blk);
      if (Kc != nullptr && Vc != nullptr) {
        const size_t poff = (static_cast<size_t>(b) * g.slots + pslot) * cblk;
        cb.add(Ly.pool_k + poff, static_cast<const char*>(Kc) + b * cblk, cblk);
        cb.add(Ly.pool_v + poff, static_cast<const char*>(Vc) + b * cblk, cblk);
      }
    }
    nx.recent_count += 1;
    nx.evicted += ev;
  }
  nx.blocks_seen += 1;
  cb.flush();
  if (cb.err != cudaSuccess) return cuda_fail(cb.err, "append copy launch");
  if (!to_sink && Kc != nullptr && Vc != nullptr) {
    const int pslot = (nx.mid_head + nx.mid_count + nx.recent_count - 1) % g.slots;
    cudaError_t e = pf::launch_kmean(Ly.pool_k, Ly.kbar, cf.batch, g.slots, g.n_c, g.HD, pslot, 1,
                                     static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "append key-mean launch");
  }
  Ly = nx;
  if (evicted) *evicted = ev;
  return PF_OK;
}

pf_status pf_cache_load_mid(pf_cache* c, int layer, const void* Kc, const void* Vc, int nblocks, int* evicted,
                            void* stream) {
  pf_status s = check_layer(c, layer);
  if (s != PF_OK) return s;
  if (nblocks < 0) return fail(PF_ERR_ARG, "nblocks < 0");
  if (nblocks == 0) {
    if (evicted) *evicted = 0;
    return PF_OK;
  }
  if ((s = check_ptr(Kc, "Kc")) != PF_OK || (s = check_ptr(Vc, "Vc")) != PF_OK) return s;
  Layer& Ly = c->L[layer];
  const pf_config& cf = c->cfg;
  const Geometry& g = c->g;
  if (Ly.sink_filled < cf.sink_blocks) return fail(PF_ERR_STATE, "load_mid needs a full sink");
  if (Ly.recent_count != 0) return fail(PF_ERR_STATE, "load_mid needs an empty recent partition");
  if (cf.mid_capacity == 0) {
    Ly.evicted += nblocks;
    Ly.blocks_seen += nblocks;
    if (evicted) *evicted = nblocks;
    return PF_OK;
  }
  const size_t cblk = static_cast<size_t>(g.n_c) * g.HD * 2;
  const int keep = nblocks < cf.mid_capacity ? nblocks : cf.mid_capacity;
  const int first = nblocks - keep;  // source blocks before this are evicted on the way
  Layer nx = Ly;
  int ev = 0;
  // place blocks first .. nblocks-1 after the live ones, evicting as needed
  const int over = nx.mid_count + keep - cf.mid_capacity;
  if (over > 0) {
    nx.mid_head = (nx.mid_head + over) % g.slots;
    nx.mid_count -= over;
  }
  ev = first + (over > 0 ? over : 0);
  const int start_slot = (nx.mid_head + nx.mid_count) % g.slots;
  CopyBuilder cb;
  cb.st = static_cast<cudaStream_t>(stream);
  for (int b = 0; b < cf.batch; ++b) {
    int i = 0;
    while (i < keep) {
      const int slot = (start_slot + i) % g.slots;
      const int run = (g.slots - slot) < (keep - i) ? (g.slots - slot) : (keep - i);
      const size_t src = (static_cast<size_t>(b) * nblocks + first + i) * cblk;
      const size_t dst = (static_cast<size_t>(b) * g.slots + slot) * cblk;
      cb.add(Ly.pool_k + dst, static_cast<const char*>(Kc) + src, run * cblk);
      cb.add(Ly.pool_v + dst, static_cast<const char*>(Vc) + src, run * cblk);
      i += run;
    }
  }
  nx.mid_count += keep;
  nx.evicted += ev;
  nx.blocks_seen += nblocks;
  nx.sel_valid = false;
  cb.flush();
  if (cb.err != cudaSuccess) return cuda_fail(cb.err, "load_mid copy launch");
  for (int i = 0; i < keep;) {
    const int slot = (start_slot + i) % g.slots;
    const int run = (g.slots - slot) < (keep - i) ? (g.slots - slot) : (keep - i);
    cudaError_t e = pf::launch_kmean(Ly.pool_k, Ly.kbar, cf.batch, g.slots, g.n_c, g.HD, slot, run,
                                     static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "load_mid key-mean launch");
    i += run;
  }
  Ly = nx;
  if (evicted) *evicted = ev;
  return PF_OK;
}

pf_status pf_select_mid_ex(pf_cache* c, int layer, const void* Q, const pf_select_opts* opts, int32_t* sel_out,
                           float* scores_out, void* stream) {
  pf_status s = check_layer(c, layer);
  if (s != PF_OK) return s;
  const pf_config& cf = c->cfg;
  const Geometry& g = c->g;
  pf_select_opts o;
  o.policy = PF_ROUTE_SCORE;
  o.q_stride = 1;
  o.head_lo = 0;
  o.head_hi = 0;
  o.heads_total = 0;
  o.scores_in = nullptr;
  if (opts != nullptr) o = *opts;
  if (o.head_lo == 0 && o.head_hi == 0) o.head_hi = cf.heads;
  if (o.policy < PF_ROUTE_SCORE || o.policy > PF_ROUTE_FIFO) return fail(PF_ERR_ARG, "unknown routing policy %d", o.policy);
  if (o.q_stride < 1) return fail(PF_ERR_ARG, "q_stride %d < 1", o.q_stride);
  if (o.q_stride > g.n) o.q_stride = g.n;  // the same rows (row 0 only); keeps n + q_stride in int
  if (o.head_lo < 0 || o.head_hi > cf.heads || o.head_lo >= o.head_hi)
    return fail(PF_ERR_ARG, "head range [%d, %d) not inside [0, %d)", o.head_lo, o.head_hi, cf.heads);
  if (o.heads_total < 0) return fail(PF_ERR_ARG, "heads_total %d < 0", o.heads_total);
  const bool scored = o.policy == PF_ROUTE_SCORE || o.policy == PF_ROUTE_SCORES_ONLY;
  if (scored && (s = check_ptr(Q, "Q")) != PF_OK) return s;
  if (o.policy == PF_ROUTE_GIVEN) {
    if (o.scores_in == nullptr) return fail(PF_ERR_ARG, "PF_ROUTE_GIVEN needs scores_in");
    if (reinterpret_cast<uintptr_t>(o.scores_in) % 4 != 0) return fail(PF_ERR_ARG, "scores_in is not 4-byte aligned");
  }
  if (o.policy == PF_ROUTE_SCORES_ONLY && scores_out == nullptr)
    return fail(PF_ERR_ARG, "PF_ROUTE_SCORES_ONLY needs scores_out");
  Layer& Ly = c->L[layer];
  const bool stores = o.policy != PF_ROUTE_SCORES_ONLY;
  if (Ly.mid_count == 0 || (stores && cf.n_top == 0)) {
    if (stores) {
      Ly.sel_valid = true;
      Ly.n_sel = 0;
    }
    return PF_OK;
  }
  pf::SelectArgs a;
  a.Q = Q;
  a.B = cf.batch;
  a.n = g.n;
  a.HD = g.HD;
  a.qsum = Ly.qsum;
  a.pool_k = Ly.pool_k;
  a.kbar = Ly.kbar;
  a.slots = g.slots;
  a.n_c = g.n_c;
  a.head = Ly.mid_head;
  a.count = Ly.mid_count;
  a.chunk_rows = g.chunk_rows;
  // query sums over 256-column slabs (128 for an odd head count) of the
  // heads used, in row chunks; then one dot product per block against its
  // mean key
  const int nslabs = (o.head_hi - o.head_lo) * pf::kHeadDim /
                     pf::select_slab_cols(o.head_lo * pf::kHeadDim, o.head_hi * pf::kHeadDim);
  a.qtot = Ly.qsum + static_cast<size_t>(cf.batch) * pf::kSelMaxRowChunks * g.HD;
  a.chunks_per_block = 1;
  a.p_stride = 1;
  a.k_stride = 1;
  a.partial_ld = g.slots;
  a.slab_ticket = Ly.ticket + cf.batch;
  {
    // row chunks per slab: as many as keep the query-sum grid within one
    // wave of two CTAs per SM
    static pf::PerDevice sm_count;
    int sms = 0;
    cudaError_t e = sm_count.get(&sms, [](int dev, int* v) {
      return cudaDeviceGetAttribute(v, cudaDevAttrMultiProcessorCount, dev);
    });
    if (e != cudaSuccess) return cuda_fail(e, "SM count");
    const long long per = 1LL * nslabs * cf.batch;
    long long R = (2LL * sms) / per;
    a.row_chunks = static_cast<int>(std::max(1LL, std::min<long long>(pf::kSelMaxRowChunks, R)));
  }
  const int rows = (g.n + o.q_stride - 1) / o.q_stride;
  const int heads_norm = o.heads_total > 0 ? o.heads_total : o.head_hi - o.head_lo;
  a.score_scale = static_cast<float>(1.0 / (static_cast<double>(rows) * heads_norm * std::sqrt(128.0)));
  a.partial = Ly.partial;
  a.scores = Ly.scores;
  a.ticket = Ly.ticket;
  a.n_top = cf.n_top;
  a.sel_slots = Ly.sel;
  a.sel_out = sel_out;
  a.scores_out = scores_out;
  a.q_stride = o.q_stride;
  a.d_lo = o.head_lo * 128;
  a.d_hi = o.head_hi * 128;
  a.topk = stores ? 1 : 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  switch (o.policy) {
    case PF_ROUTE_SCORE:
    case PF_ROUTE_SCORES_ONLY:
      e = pf::launch_select_cached(a, st);
      break;
    case PF_ROUTE_GIVEN:
      a.partial = const_cast<float*>(o.scores_in);
      a.partial_ld = Ly.mid_count;
      a.chunks_per_block = 1;
      a.p_stride = 1;
      a.k_stride = 1;
      a.score_scale = 1.f;
      e = pf::launch_topk_given(a, st);
      break;
    default:
      e = pf::launch_select_fifo(a, st);
      break;
  }
  if (e != cudaSuccess) return cuda_fail(e, "select launch");
  if (stores) {
    Ly.sel_valid = true;
    Ly.n_sel = cf.n_top < Ly.mid_count ? cf.n_top : Ly.mid_count;
  }
  return PF_OK;
}

pf_status pf_select_mid(pf_cache* c, int layer, const void* Q, int32_t* sel_out, float* scores_out, void* stream) {
  return pf_select_mid_ex(c, layer, Q, nullptr, sel_out, scores_out, stream);
}

pf_status pf_rope_shift(pf_cache* c, int layer, unsigned parts, int delta, void* stream) {
  if (c == nullptr) return fail(PF_ERR_ARG, "cache is NULL");
  if (layer != -1) {
    pf_status s = check_layer(c, layer);
    if (s != PF_OK) return s;
  }
  if (parts & ~(PF_PART_SINK | PF_PART_MID | PF_PART_RECENT)) return fail(PF_ERR_ARG, "unknown partition bits");
  const pf_config& cf = c->cfg;
  const Geometry& g = c->g;
  RunBuilder rb, rm;
  rb.st = static_cast<cudaStream_t>(stream);
  rm.st = rb.st;
  rm.f32 = true;
  rb.tab.pairs = cf.rope_split[0] / 2;
  for (int k = 0; k < 32; ++k) {
    rb.tab.c[k] = 1.f;
    rb.tab.s[k] = 0.f;
  }
  for (int k = 0; k < rb.tab.pairs; ++k) {
    const double theta = std::pow(static_cast<double>(cf.rope_base), -2.0 * k / cf.rope_split[0]);
    const double ang = theta * static_cast<double>(delta);
    rb.tab.c[k] = static_cast<float>(std::cos(ang));
    rb.tab.s[k] = static_cast<float>(std::sin(ang));
  }
  rm.tab = rb.tab;
  if (delta == 0 || parts == 0) return PF_OK;
  const int l0 = layer < 0 ? 0 : layer, l1 = layer < 0 ? cf.layers : layer + 1;
  const long long H = cf.heads;
  const size_t rowb = static_cast<size_t>(g.HD) * 2;
  const bool sink_lazy = cf.sink_rope_in_attention != 0;
  if ((parts & PF_PART_SINK) && sink_lazy)
    for (int l = l0; l < l1; ++l)
      if (c->L[l].sink_filled < cf.sink_blocks)
        return fail(PF_ERR_STATE, "layer %d: the sink shift is applied in attention and needs a full sink (%d of %d "
                    "blocks)", l, c->L[l].sink_filled, cf.sink_blocks);
  for (int l = l0; l < l1; ++l) {
    Layer& Ly = c->L[l];
    if ((parts & PF_PART_SINK) && !sink_lazy) {
      if (Ly.sink_filled == cf.sink_blocks) {
        rb.add(Ly.sink_k, 1LL * cf.batch * cf.sink_blocks * g.n * H);
      } else {
        for (int b = 0; b < cf.batch; ++b)
          rb.add(Ly.sink_k + static_cast<size_t>(b) * cf.sink_blocks * g.n * rowb, 1LL * Ly.sink_filled * g.n * H);
      }
    }
    auto add_ring = [&](char* base, int slots, int head, int count, long long rows_per_slot) {
      for (int b = 0; b < cf.batch; ++b) {
        int i = 0;
        while (i < count) {
          const int slot = (head + i) % slots;
          const int run = (slots - slot) < (count - i) ? (slots - slot) : (count - i);
          rb.add(base + (static_cast<size_t>(b) * slots + slot) * rows_per_slot * rowb, run * rows_per_slot * H);
          i += run;
        }
      }
    };
    if (parts & PF_PART_MID) add_ring(Ly.pool_k, g.slots, Ly.mid_head, Ly.mid_count, g.n_c);
    if (parts & PF_PART_RECENT) {
      add_ring(Ly.recent_k, cf.recent_blocks, Ly.recent_head, Ly.recent_count, g.n);
      if (cf.mid_capacity > 0)
        add_ring(Ly.pool_k, g.slots, (Ly.mid_head + Ly.mid_count) % g.slots, Ly.recent_count, g.n_c);
    }
    // the cached mean keys rotate with their blocks (the mean of rotated keys
    // is the rotated mean)
    auto add_mean_ring = [&](int head, int count) {
      for (int b = 0; b < cf.batch; ++b) {
        int i = 0;
        while (i < count) {
          const int slot = (head + i) % g.slots;
          const int run = (g.slots - slot) < (count - i) ? (g.slots - slot) : (count - i);
          rm.add(Ly.kbar + (static_cast<size_t>(b) * g.slots + slot) * g.HD, 1LL * run * H);
          i += run;
        }
      }
    };
    if (parts & PF_PART_MID) add_mean_ring(Ly.mid_head, Ly.mid_count);
    if ((parts & PF_PART_RECENT) && cf.mid_capacity > 0)
      add_mean_ring((Ly.mid_head + Ly.mid_count) % g.slots, Ly.recent_count);
  }
  rb.flush();
  rm.flush();
  if (rb.err != cudaSuccess) return cuda_fail(rb.err, "rope shift launch");
  if (rm.err != cudaSuccess) return cuda_fail(rm.err, "rope shift (mean keys) launch");
  if (parts & PF_PART_SINK)
    for (int l = l0; l < l1; ++l) c->L[l].total_shift += delta;
  return PF_OK;
}

pf_status pf_attend_tail_plan(long long full_units, int tails, int n_tiles, int sms, int* big, int* small,
                              int* split) {
  if (big == nullptr || small == nullptr || split == nullptr) return fail(PF_ERR_ARG, "null output");
  if (full_units < 0 || tails < 0 || n_tiles < 0 || sms < 1) return fail(PF_ERR_ARG, "negative size or sms < 1");
  const pf::TailPlan tp = pf::attend_tail_plan(full_units, tails, n_tiles, sms);   // tp.group stays internal
  *big = tp.big;
  *small = tp.small;
  *split = tp.split;
  return PF_OK;
}

pf_status pf_attend(pf_cache* c, int layer, const void* Q, const void* K_cur, const void* V_cur, void* O, float* lse,
                    void* stream) {
  pf_status s = check_layer(c, layer);
  if (s != PF_OK) return s;
  if ((s = check_ptr(Q, "Q")) != PF_OK || (s = check_ptr(K_cur, "K_cur")) != PF_OK ||
      (s = check_ptr(V_cur, "V_cur")) != PF_OK || (s = check_ptr(O, "O")) != PF_OK)
    return s;
  if (O == Q || O == K_cur || O == V_cur) return fail(PF_ERR_ARG, "O must not alias the inputs");
  if (lse != nullptr && reinterpret_cast<uintptr_t>(lse) % 4 != 0) return fail(PF_ERR_ARG, "lse misaligned");
  Layer& Ly = c->L[layer];
  const pf_config& cf = c->cfg;
  const Geometry& g = c->g;
  pf::AttendParams p;
  std::memset(&p, 0, sizeof(p));
  int n_sel = 0;
  const int32_t* sel = nullptr;
  if (cf.n_top >= Ly.mid_count) {
    n_sel = Ly.mid_count;  // every live block
  } else if (Ly.sel_valid) {
    n_sel = Ly.n_sel;
    sel = Ly.sel;
  } else {
    return fail(PF_ERR_STATE, "layer %d: the pool has %d blocks > n_top and no current selection (call pf_select_mid)",
                layer, Ly.mid_count);
  }
  const int B = cf.batch, H = cf.heads;
  const int sink_rows = Ly.sink_filled * g.n;
  if (!Ly.maps_ready) {
    // the arena's partitions: encoded once per layer
    if (cf.sink_blocks > 0) {
      if ((s = encode_map(&Ly.tm_k[0], Ly.sink_k, H, 1LL * cf.sink_blocks * g.n, B, 32)) != PF_OK) return s;
      if ((s = encode_map(&Ly.tm_v[0], Ly.sink_v, H, 1LL * cf.sink_blocks * g.n, B, 32)) != PF_OK) return s;
    }
    if ((s = encode_map(&Ly.tm_k[1], Ly.pool_k, H, g.n_c, 1LL * B * g.slots, 32)) != PF_OK) return s;
    if ((s = encode_map(&Ly.tm_v[1], Ly.pool_v, H, g.n_c, 1LL * B * g.slots, 32)) != PF_OK) return s;
    if ((s = encode_map(&Ly.tm_k[2], Ly.recent_k, H, g.n, 1LL * B * cf.recent_blocks, 32)) != PF_OK) return s;
    if ((s = encode_map(&Ly.tm_v[2], Ly.recent_v, H, g.n, 1LL * B * cf.recent_blocks, 32)) != PF_OK) return s;
    Ly.maps_ready = true;
  }
  // the caller's tensors: encoded per call
  if ((s = encode_map(&p.tm_q, Q, H, g.n, B, 128)) != PF_OK) return s;
  if ((s = encode_map(&p.tm_k[pf::kPartCur], K_cur, H, g.n, B, 32)) != PF_OK) return s;
  if ((s = encode_map(&p.tm_v[pf::kPartCur], V_cur, H, g.n, B, 32)) != PF_OK) return s;
  if (cf.sink_blocks > 0) {
    p.tm_k[pf::kPartSink] = Ly.tm_k[0];
    p.tm_v[pf::kPartSink] = Ly.tm_v[0];
  } else {
    p.tm_k[pf::kPartSink] = p.tm_k[pf::kPartCur];
    p.tm_v[pf::kPartSink] = p.tm_v[pf::kPartCur];
  }
  p.tm_k[pf::kPartMid] = Ly.tm_k[1];
  p.tm_v[pf::kPartMid] = Ly.tm_v[1];
  p.tm_k[pf::kPartRecent] = Ly.tm_k[2];
  p.tm_v[pf::kPartRecent] = Ly.tm_v[2];
  p.O = O;
  p.lse = lse;
  p.B = B;
  p.H = H;
  p.n = g.n;
  p.n_c = g.n_c;
  p.sink_rows = sink_rows;
  p.n_sel = n_sel;
  p.sel_slots = sel;
  p.sel_stride = cf.n_top;
  p.mid_head = Ly.mid_head;
  p.pool_slots = g.slots;
  p.n_recent = Ly.recent_count;
  p.recent_head = Ly.recent_head;
  p.recent_slots = cf.recent_blocks;
  p.sb_sink = (sink_rows + 31) / 32;
  p.sb_mid = (g.n_c + 31) / 32;
  p.sb_blk = (g.n + 31) / 32;
  p.n_sub = p.sb_sink + n_sel * p.sb_mid + p.n_recent * p.sb_blk + p.sb_blk;
  p.n_tiles = (p.n_sub + 3) / 4;
  p.sb_mid_lo = p.sb_sink;
  p.sb_mid_hi = p.sb_sink + n_sel * p.sb_mid;
  p.exact = (sink_rows % 32 == 0 && g.n % 32 == 0) ? 1 : 0;
  p.q_tiles = (g.n + 127) / 128;
  p.part_o = c->part_o;
  p.part_ml = c->part_ml;
  p.rotate_sink = (cf.sink_rope_in_attention && Ly.total_shift != 0 && sink_rows > 0) ? 1 : 0;
  p.sink_rope.pairs = cf.rope_split[0] / 2;
  for (int k = 0; k < 32; ++k) {
    p.sink_rope.c[k] = 1.f;
    p.sink_rope.s[k] = 0.f;
  }
  for (int k = 0; k < p.sink_rope.pairs; ++k) {
    const double theta = std::pow(static_cast<double>(cf.rope_base), -2.0 * k / cf.rope_split[0]);
    const double ang = theta * static_cast<double>(Ly.total_shift);
    p.sink_rope.c[k] = static_cast<float>(std::cos(ang));
    p.sink_rope.s[k] = static_cast<float>(std::sin(ang));
  }
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(128.0));
  p.err = c->err;
  p.timeout_cycles = c->timeout_cycles;
  const long long units = 1LL * B * H * p.q_tiles;
  if (units > 0x7fffffffLL) return fail(PF_ERR_CAPACITY, "too many work units");
  cudaError_t e = pf::launch_attend(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "attend launch");
  return PF_OK;
}

pf_status pf_attend_step(pf_cache* c, int layer, int step, const void* Q, const void* K_cur, const void* V_cur,
                         void* O, float* lse, void* stream) {
  pf_status s = check_layer(c, layer);
  if (s != PF_OK) return s;
  if (step < 0) return fail(PF_ERR_ARG, "step %d < 0", step);
  if (step == 0) {
    // check attention's arguments first, so a refused call selects nothing
    if ((s = check_ptr(Q, "Q")) != PF_OK || (s = check_ptr(K_cur, "K_cur")) != PF_OK ||
        (s = check_ptr(V_cur, "V_cur")) != PF_OK || (s = check_ptr(O, "O")) != PF_OK)
      return s;
    if (O == Q || O == K_cur || O == V_cur) return fail(PF_ERR_ARG, "O must not alias the inputs");
    if (lse != nullptr && reinterpret_cast<uintptr_t>(lse) % 4 != 0) return fail(PF_ERR_ARG, "lse misaligned");
    if ((s = pf_select_mid(c, layer, Q, nullptr, nullptr, stream)) != PF_OK) return s;
  }
  return pf_attend(c, layer, Q, K_cur, V_cur, O, lse, stream);
}

pf_status pf_finish_block(pf_cache* c, const void* const* K, const void* const* V, const void* const* Kc,
                          const void* const* Vc, int* evicted, void* stream) {
  if (c == nullptr) return fail(PF_ERR_ARG, "cache is NULL");
  if (K == nullptr || V == nullptr) return fail(PF_ERR_ARG, "K and V arrays must not be NULL");
  const pf_config& cf = c->cfg;
  pf_status s;
  for (int l = 0; l < cf.layers; ++l) {
    if ((s = check_ptr(K[l], "K[layer]")) != PF_OK || (s = check_ptr(V[l], "V[layer]")) != PF_OK) return s;
    const Layer& Ly = c->L[l];
    if (Ly.sink_filled < cf.sink_blocks || cf.mid_capacity == 0) continue;   // Kc/Vc not needed
    if (Kc == nullptr || Vc == nullptr) return fail(PF_ERR_ARG, "Kc and Vc arrays must not be NULL");
    if ((s = check_ptr(Kc[l], "Kc[layer]")) != PF_OK || (s = check_ptr(Vc[l], "Vc[layer]")) != PF_OK) return s;
  }
  int ev0 = 0;
  for (int l = 0; l < cf.layers; ++l) {
    int ev = 0;
    s = pf_cache_append_block(c, l, K[l], V[l], Kc ? Kc[l] : nullptr, Vc ? Vc[l] : nullptr, &ev, stream);
    if (s != PF_OK) return s;
    if (l == 0) ev0 = ev;
    else if (ev != ev0) return fail(PF_ERR_STATE, "layer %d evicted %d blocks, layer 0 %d", l, ev, ev0);
  }
  if (ev0 > 0 && (s = pf_rope_shift(c, -1, PF_PART_SINK, ev0 * cf.block_frames, stream)) != PF_OK) return s;
  if (evicted) *evicted = ev0;
  return PF_OK;
}

// Saved host state: a header (magic, version, the configuration) and one
// record per layer.
namespace {
constexpr uint32_t kStateMagic = 0x50465354u;   // "PFST"
constexpr uint32_t kStateVersion = 1;
struct StateHeader {
  uint32_t magic, version;
  pf_config cfg;
};
struct LayerState {
  int32_t blocks_seen, sink_filled, recent_count, recent_head, mid_count, mid_head, sel_valid, n_sel;
  int64_t evicted, total_shift;
};
}  // namespace

pf_status pf_cache_state_bytes(const pf_cache* c, size_t* bytes) {
  if (c == nullptr || bytes == nullptr) return fail(PF_ERR_ARG, "cache and bytes must not be NULL");
  *bytes = sizeof(StateHeader) + sizeof(LayerState) * static_cast<size_t>(c->cfg.layers);
  return PF_OK;
}

pf_status pf_cache_save_state(const pf_cache* c, void* buf, size_t bytes) {
  size_t need = 0;
  pf_status s = pf_cache_state_bytes(c, &need);
  if (s != PF_OK) return s;
  if (buf == nullptr || bytes < need) return fail(PF_ERR_ARG, "state buffer of %zu bytes, %zu needed", bytes, need);
  StateHeader h;
  std::memset(&h, 0, sizeof(h));
  h.magic = kStateMagic;
  h.version = kStateVersion;
  h.cfg = c->cfg;
  char* out = static_cast<char*>(buf);
  std::memcpy(out, &h, sizeof(h));
  out += sizeof(h);
  for (const Layer& Ly : c->L) {
    LayerState r;
    std::memset(&r, 0, sizeof(r));
    r.blocks_seen = Ly.blocks_seen;
    r.sink_filled = Ly.sink_filled;
    r.recent_count = Ly.recent_count;
    r.recent_head = Ly.recent_head;
    r.mid_count = Ly.mid_count;
    r.mid_head = Ly.mid_head;
    r.sel_valid = Ly.sel_valid ? 1 : 0;
    r.n_sel = Ly.n_sel;
    r.evicted = Ly.evicted;
    r.total_shift = Ly.total_shift;
    std::memcpy(out, &r, sizeof(r));
    out += sizeof(r);
  }
  return PF_OK;
}

pf_status pf_cache_load_state(pf_cache* c, const void* buf, size_t bytes) {
  size_t need = 0;
  pf_status s = pf_cache_state_bytes(c, &need);
  if (s != PF_OK) return s;
  if (buf == nullptr || bytes != need) return fail(PF_ERR_ARG, "state of %zu bytes, %zu expected", bytes, need);
  const char* in = static_cast<const char*>(buf);
  StateHeader h;
  std::memcpy(&h, in, sizeof(h));
  in += sizeof(h);
  if (h.magic != kStateMagic || h.version != kStateVersion) return fail(PF_ERR_ARG, "not a saved cache state");
  if (std::memcmp(&h.cfg, &c->cfg, sizeof(pf_config)) != 0)
    return fail(PF_ERR_STATE, "the state was saved from a cache with another configuration");
  const pf_config& cf = c->cfg;
  std::vector<LayerState> rs(static_cast<size_t>(cf.layers));
  for (int l = 0; l < cf.layers; ++l) {
    LayerState& r = rs[static_cast<size_t>(l)];
    std::memcpy(&r, in, sizeof(r));
    in += sizeof(r);
    const int cap = cf.mid_capacity;
    const bool okay = r.blocks_seen >= 0 && r.sink_filled >= 0 && r.sink_filled <= cf.sink_blocks &&
                      r.recent_count >= 0 && r.recent_count <= cf.recent_blocks && r.recent_head >= 0 &&
                      r.recent_head < cf.recent_blocks && r.mid_count >= 0 && r.mid_count <= cap &&
                      r.mid_head >= 0 && r.mid_head < c->g.slots && (r.sel_valid == 0 || r.sel_valid == 1) &&
                      r.n_sel >= 0 && r.n_sel <= cf.n_top && r.n_sel <= r.mid_count && r.evicted >= 0 &&
                      (r.sink_filled == cf.sink_blocks || (r.recent_count == 0 && r.mid_count == 0));
    if (!okay) return fail(PF_ERR_STATE, "layer %d of the saved state is outside the configuration's limits", l);
  }
  for (int l = 0; l < cf.layers; ++l) {
    const LayerState& r = rs[static_cast<size_t>(l)];
    Layer& Ly = c->L[l];
    Ly.blocks_seen = r.blocks_seen;
    Ly.sink_filled = r.sink_filled;
    Ly.recent_count = r.recent_count;
    Ly.recent_head = r.recent_head;
    Ly.mid_count = r.mid_count;
    Ly.mid_head = r.mid_head;
    Ly.sel_valid = r.sel_valid != 0;
    Ly.n_sel = r.n_sel;
    Ly.evicted = r.evicted;
    Ly.total_shift = r.total_shift;
  }
  return PF_OK;
}

pf_status pf_poll_device_error(pf_cache* c, void* stream, unsigned* code) {
  if (c == nullptr) return fail(PF_ERR_ARG, "cache is NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned w = 0;
  e = cudaMemcpy(&w, c->err, sizeof(w), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read error word");
  if (code) *code = w;
  if (w != 0) {
    e = cudaMemset(c->err, 0, sizeof(unsigned));
    if (e != cudaSuccess) return cuda_fail(e, "clear error word");
    return fail(PF_ERR_TIMEOUT, "a device-side wait gave up (site 0x%x)", w);
  }
  return PF_OK;
}

pf_status pf_selftest_wait_timeout(pf_cache* c, unsigned timeout_us, void* stream) {
  if (c == nullptr) return fail(PF_ERR_ARG, "cache is NULL");
  if (timeout_us == 0 || timeout_us > 10u * 1000u * 1000u) return fail(PF_ERR_ARG, "timeout_us must be in (0, 1e7]");
  int dev = 0, khz = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&khz, cudaDevAttrClockRate, dev);
  if (khz <= 0) khz = 2000000;
  const long long cycles = static_cast<long long>(timeout_us) * (khz / 1000);
  cudaError_t e = pf::launch_wait_timeout_selftest(c->err, cycles, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
  return PF_OK;
}

}  // extern "C"
