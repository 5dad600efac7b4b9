// pf_internal.h -- launch interfaces between the host state machine
// (pf_cache.cpp) and the kernels.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

namespace pf {

constexpr int kHeadDim = 128;
constexpr int kMaxSegs = 64;
constexpr int kMaxDevices = 64;

// A launcher's per-device set-up (a kernel attribute raised, a grid size
// from the device's SM count and the kernel's occupancy), done once per
// device, with that device current, under a lock.  A process may drive
// several GPUs from several threads.  The cached results belong to the
// device's primary context: after cudaDeviceReset they are stale.
class PerDevice {
 public:
  // *out = the value compute(dev, &value) produced for the current device.
  template <class F>
  cudaError_t get(int* out, F compute) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu_);
    if (!done_[dev]) {
      int v = 0;
      e = compute(dev, &v);
      if (e != cudaSuccess) return e;
      value_[dev] = v;
      done_[dev] = true;
    }
    *out = value_[dev];
    return cudaSuccess;
  }

 private:
  std::mutex mu_;
  int value_[kMaxDevices] = {};
  bool done_[kMaxDevices] = {};
};

// SMs x resident CTAs of `kernel` (256 threads, no dynamic shared memory)
// on device dev: a grid that fills the GPU in one wave.
template <class K>
cudaError_t one_wave_grid(K kernel, int dev, int* out) {
  int sms = 0, per_sm = 0;
  cudaError_t e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, 256, 0);
  if (e != cudaSuccess) return e;
  *out = sms * (per_sm > 0 ? per_sm : 1);
  return cudaSuccess;
}

// Device error codes written to the cache's error word.
constexpr unsigned kDevErrTimeoutBase = 0x100u;  // | site id

// ------------------------------------------------------------- RoPE shift
// A list of contiguous runs of "row-heads" (one head's 128-dim key vector,
// 256 bytes), start[] = prefix sums of the run lengths.
struct RowRuns {
  int n;
  long long start[kMaxSegs + 1];
  void* ptr[kMaxSegs];
};

struct RopeTable {
  int pairs;  // rotary pairs to rotate (rope_split[0] / 2)
  float c[32];
  float s[32];
};

#ifdef __CUDACC__
// Rotate the rotary pairs held in 16-byte word `word` (bf16 pairs 4 word ..
// 4 word + 3) of a key vector: (re, im) -> (re c - im s, re s + im c) in
// float32, rounded to bf16 (nearest even); cs / sn hold the four pairs'
// cosines and sines.  Pairs at or past `pairs` stay.  Shared by the
// in-place shift and the shift applied inside attention, so both round
// identically.
__device__ __forceinline__ void rope_rotate_word_cs(uint4& w, int word, int pairs, const float* cs,
                                                    const float* sn) {
  uint32_t v[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    if (word * 4 + q < pairs) {
      const float re = __uint_as_float(v[q] << 16), im = __uint_as_float(v[q] & 0xffff0000u);
      const float nre = re * cs[q] - im * sn[q];
      const float nim = re * sn[q] + im * cs[q];
      uint32_t r;
      asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(nim), "f"(nre));
      v[q] = r;
    }
  }
  w = make_uint4(v[0], v[1], v[2], v[3]);
}

__device__ __forceinline__ void rope_rotate_word(uint4& w, int word, const RopeTable& t) {
  float cs[4], sn[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int pair = (word * 4 + q) & 31;
    cs[q] = t.c[pair];
    sn[q] = t.s[pair];
  }
  rope_rotate_word_cs(w, word, t.pairs, cs, sn);
}
#endif

// bf16 key vectors, in place.
cudaError_t launch_rope_shift(const RowRuns& runs, const RopeTable& tab, cudaStream_t st);
// The same rotation of float32 128-dim vectors (cached mean keys); runs count vectors.
cudaError_t launch_rope_shift_f32(const RowRuns& runs, const RopeTable& tab, cudaStream_t st);

// ------------------------------------------------------------- copies
// start[] = prefix sums of run lengths in 16-byte units.
struct CopyRuns {
  int n;
  long long start[kMaxSegs + 1];
  void* dst[kMaxSegs];
  const void* src[kMaxSegs];
};

cudaError_t launch_copy(const CopyRuns& runs, cudaStream_t st);

// ------------------------------------------------------------- selection
// The cache path's query sums run over slabs of 256 columns of the H * D
// query vector (128 when the score's column range is an odd number of
// heads), in at most kSelMaxRowChunks chunks of query rows per slab.
// kSelSlabCols is the narrowest slab (it sizes the slab tickets).
constexpr int kSelSlabCols = 128;
constexpr int kSelMaxRowChunks = 32;
inline int select_slab_cols(int d_lo, int d_hi) { return ((d_hi - d_lo) % 256 == 0) ? 256 : 128; }

struct SelectArgs {
  const void* Q;        // [B, n, H, D] bf16
  int B, n, HD;         // HD = H * D
  float* qsum;          // [B, HD] query sums (streaming path); [B, kSelMaxRowChunks, HD]
                        // per-row-chunk partial sums (cache path)
  float* qtot;          // cache path: [B, HD] the chunks' sums added
  unsigned* slab_ticket;  // cache path: [B, HD / kSelSlabCols], zero on entry, left zero on exit
  int row_chunks;       // cache path: row chunks per slab (1 .. kSelMaxRowChunks)
  const void* pool_k;   // [B, slots, n_c, H, D] bf16
  const float* kbar;    // [B, slots, HD] mean key per pool slot, or null: stream pool_k
  int slots, n_c;
  int head, count;      // live blocks: age p -> slot (head + p) % slots
  int chunk_rows;       // pool rows per scoring CTA
  int chunks_per_block;
  float score_scale;    // 1 / (n * n_c * H * sqrt(D))
  float* partial;       // partial scores: element (block age q, part k) of batch item b at
                        // b * partial_ld + q * p_stride + k * k_stride, k < chunks_per_block
  int p_stride, k_stride;
  float* scores;        // [B, slots] by age
  unsigned* ticket;     // [B], zero on entry, left zero on exit
  int n_top;
  int32_t* sel_slots;   // [B, n_top] pool slots, ascending age
  int32_t* sel_out;     // optional [B, k] ages
  float* scores_out;    // optional [B, count]
  int q_stride;         // query rows 0, q_stride, 2 q_stride, ... are pooled
  int d_lo, d_hi;       // elements [d_lo, d_hi) of a token's H * D vector enter the score
  int topk;             // 0: write the scores only (no selection)
  int partial_ld;       // per-batch-item length of `partial`
};

// qpool + scoring of the streamed compressed keys (+ top-k unless a.topk == 0).
cudaError_t launch_select(const SelectArgs& a, cudaStream_t st);
// The same from the cached mean keys (a.kbar): query sums per slab, then one
// dot product per block and the top-k (unless a.topk == 0), two kernels.
cudaError_t launch_select_cached(const SelectArgs& a, cudaStream_t st);
// Top-k of given scores: a.partial holds [B, partial_ld] scores by age
// (chunks_per_block = 1, score_scale = 1).
cudaError_t launch_topk_given(const SelectArgs& a, cudaStream_t st);
// The min(n_top, count) most recent live blocks.
cudaError_t launch_select_fifo(const SelectArgs& a, cudaStream_t st);

// kbar[b, slot] = mean of the block's n_c keys, slots [slot0, slot0 + nslots).
cudaError_t launch_kmean(const void* pool_k, float* kbar, int B, int slots, int n_c, int HD, int slot0, int nslots,
                         cudaStream_t st);

// ------------------------------------------------------------- attention
// Partition ids of the K/V tensor maps.
enum { kPartSink = 0, kPartMid = 1, kPartRecent = 2, kPartCur = 3 };

struct AttendParams {
  CUtensorMap tm_q;     // Q  (D, H, n, B)
  CUtensorMap tm_k[4];  // sink (D,H,S*n,B), mid (D,H,n_c,B*slots), recent (D,H,n,B*R), cur (D,H,n,B)
  CUtensorMap tm_v[4];
  void* O;              // [B, n, H, D] bf16
  float* lse;           // optional [B, H, n]
  int B, H, n, n_c;
  int sink_rows;        // filled sink rows per batch item
  int n_sel;            // mid blocks routed
  const int32_t* sel_slots;  // [B, sel_stride] pool slots, or null: all live blocks
  int sel_stride;
  int mid_head, pool_slots;
  int n_recent, recent_head, recent_slots;
  int sb_sink, sb_mid, sb_blk;  // 32-row sub-boxes: sink total, per mid block, per full block
  int n_sub, n_tiles;   // sub-boxes holding keys; 128-key tiles (n_sub padded to 4)
  int sb_mid_lo, sb_mid_hi;  // sub-box range of the mid blocks
  int exact;            // sink rows and block rows are multiples of 32: only mid blocks and
                        // the padding after the last key have partial sub-boxes
  int q_tiles;          // 128-row query tiles per (b, h)
  int tail_chunks;      // context chunks each ragged last query tile is split into (1 = not split)
  int tail_big, tail_small;  // of them: the first tail_big cover K/V tiles [0, tail_split) in equal
  int tail_split;            // parts, the other tail_small cover [tail_split, n_tiles) (set by launch_attend)
  int group_bh;              // (b, h) per unit group: their pairs, then their tiles' big chunks
  float* part_o;        // [tails * tail_chunks, 128, 128] unnormalised partial outputs
  float* part_ml;       // [tails * tail_chunks, 2, 128] partial row max / row sum
  int rotate_sink;      // 1: rotate the sink keys' temporal pairs by sink_rope as they are loaded
  RopeTable sink_rope;  // e^{i theta_k total_shift}
  float scale_log2;     // log2(e) / sqrt(D)
  unsigned* err;
  long long timeout_cycles;
};

// Scratch for split tails, in the cache arena: kAttendMaxTailSlots chunk
// slots of partial outputs and row statistics.
constexpr int kAttendMaxTailSlots = 256;
constexpr int kAttendMaxChunksPerTail = 16;
constexpr size_t kAttendPartOBytes = size_t(kAttendMaxTailSlots) * 128 * 128 * 4;
constexpr size_t kAttendPartMLBytes = size_t(kAttendMaxTailSlots) * 2 * 128 * 4;
// How the T ragged tiles of a launch are cut along the context (n K/V tiles
// each), given F = T P full units (P query-tile pairs per (b, h)) and `sms`
// SMs.  The (b, h) are grouped, as many as a wave's pairs take (group =
// sms / P), so that a group's ragged tiles are read alongside its pairs:
// big chunks that the SMs a group's pairs leave idle finish alongside them,
// then about one small chunk per SM for the rest.  {big, small, split, group}.
struct TailPlan {
  int big, small, split;
  int group;   // (b, h) whose query-tile pairs and big tail chunks are ordered together
};
TailPlan attend_tail_plan(long long F, int T, int n, int sms);

cudaError_t launch_attend(const AttendParams& p, cudaStream_t st);

// cuTensorMapEncodeTiled through the runtime's driver entry point (element
// strides 1, no interleave, out-of-bounds elements read as zero);
// CUDA_ERROR_NOT_SUPPORTED if the driver does not provide it.
CUresult encode_tiled(CUtensorMap* m, CUtensorMapDataType dtype, int rank, void* base, const cuuint64_t* dims,
                      const cuuint64_t* strides, const cuuint32_t* box, CUtensorMapSwizzle swizzle,
                      CUtensorMapL2promotion l2);

// Record a failure message for pf_last_error() and return the status.
int report_error(int status, const char* fmt, ...);

// ------------------------------------------------------------- self-test
cudaError_t launch_wait_timeout_selftest(unsigned* err, long long timeout_cycles, cudaStream_t st);

}  // namespace pf
