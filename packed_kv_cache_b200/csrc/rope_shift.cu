// rope_shift.cu -- incremental temporal RoPE adjustment of cached keys.
//
// PackForcing (arXiv), "Incremental RoPE adjustment": after evicting D mid
// blocks, the cached keys' temporal rotary components are multiplied by
// e^{i theta_t delta} (delta = D * B_f frames), leaving the height and width
// components alone ("1_h, 1_w").  Each 128-dim key vector of one head holds
// the temporal pairs in dims 0 .. rope_split[0]-1 as adjacent (re, im) pairs.
//
// HBM-bound.  Per key vector and head ("row") the first NW = ceil(pairs / 4)
// 16-byte words are read and written (6 words = 96 bytes for 22 pairs);
// the other 160 bytes of the row are never touched.  Each run of rows
// (a contiguous stretch of one partition) gets a 2-D tensor map
// (128 dims x rows, 256-byte row pitch).  A persistent CTA walks its tiles
// of 128 rows through a ring of shared-memory stages: TMA loads the tile's
// NW-word prefix of every row (a 96-byte-wide box), the threads rotate the
// pairs in shared memory, and TMA stores the box back in place.  The loads
// of the next six tiles are in flight while one tile is rotated and the
// previous one is stored, so DRAM always has requests queued without one
// thread per row waiting on its own loads.
#include <cuda_bf16.h>

#include "pf_internal.h"
#include "ptx.cuh"

namespace pf {

namespace {

constexpr int kRopeThreads = 256;
constexpr int kRopeRows = 128;     // rows per tile (the TMA box height)
constexpr int kRopeStages = 8;     // shared-memory ring depth
constexpr int kRopeLookahead = kRopeStages - 2;   // loads in flight ahead of the tile being rotated

struct RopeTmaArgs {
  CUtensorMap map[kMaxSegs];       // one per run: (128 dims, rows), box (8 NW, kRopeRows)
  long long tile_start[kMaxSegs + 1];
  int n;                           // runs
  RopeTable tab;
  unsigned* err;                   // device error word (timeouts), may be null
  long long timeout_cycles;
};

template <int NW>
__host__ __device__ constexpr uint32_t rope_tile_bytes() {
  return static_cast<uint32_t>(kRopeRows) * NW * 16;
}

template <int NW>
__host__ __device__ constexpr size_t rope_smem_bytes() {
  return static_cast<size_t>(kRopeStages) * rope_tile_bytes<NW>() + kRopeStages * sizeof(uint64_t);
}

template <int NW>
__global__ void __launch_bounds__(kRopeThreads, 2) rope_shift_tma_kernel(const __grid_constant__ RopeTmaArgs a) {
  constexpr uint32_t kTile = rope_tile_bytes<NW>();
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kRopeStages * kTile);
  __shared__ int abort_flag;

  const long long ntiles = a.tile_start[a.n];
  if (static_cast<long long>(blockIdx.x) >= ntiles) return;
  const long long mine = (ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x;   // tiles of this CTA
  const int tid = threadIdx.x;
  if (tid == 0) {
    for (int s = 0; s < kRopeStages; ++s) mbar_init(&full[s], 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  // thread 0 issues every copy; the run of a tile is found by a forward scan
  // (this CTA's tiles come in increasing order)
  int run_ld = 0, run_st = 0;
  auto tile_of = [&](long long k, int& run, int& row0) {
    const long long t = blockIdx.x + k * static_cast<long long>(gridDim.x);
    while (t >= a.tile_start[run + 1]) ++run;
    row0 = static_cast<int>((t - a.tile_start[run]) * kRopeRows);
  };
  auto issue_load = [&](long long k) {
    int row0;
    tile_of(k, run_ld, row0);
    const int s = static_cast<int>(k % kRopeStages);
    mbar_arrive_expect_tx(&full[s], kTile);
    tma_load_2d(smem + s * kTile, &a.map[run_ld], &full[s], 0, row0);
  };

  long long issued = 0;
  if (tid == 0) {
    for (; issued < kRopeLookahead && issued < mine; ++issued) issue_load(issued);
  }
  long long k = 0;
  for (; k < mine; ++k) {
    const int s = static_cast<int>(k % kRopeStages);
    if (tid == 0 && issued < mine) {
      // the stage of tile k + lookahead last held tile k - 2, whose store
      // must have finished reading it (the store of tile k - 1 may still)
      bulk_wait_group_read<1>();
      issue_load(issued++);
    }
    const bool ok = mbar_wait_bounded(&full[s], static_cast<uint32_t>((k / kRopeStages) & 1), &abort_flag, a.err,
                                      kDevErrTimeoutBase | 0x20u, a.timeout_cycles);
    if (!__syncthreads_and(ok)) break;
    uint4* tile = reinterpret_cast<uint4*>(smem + s * kTile);
    // word i of the tile: row i / NW, 16-byte word i % NW (consecutive
    // threads touch consecutive words: no bank conflicts)
#pragma unroll
    for (int i = tid; i < kRopeRows * NW; i += kRopeThreads) {
      uint4 w = tile[i];
      rope_rotate_word(w, i % NW, a.tab);
      tile[i] = w;
    }
    fence_proxy_async_smem();   // the rotated words, visible to the TMA store
    __syncthreads();
    if (tid == 0) {
      int row0;
      tile_of(k, run_st, row0);
      tma_store_2d(&a.map[run_st], smem + s * kTile, 0, row0);
      bulk_commit_group();
    }
  }
  if (tid == 0) {
    // a wait that gave up: let the loads still in flight land before exit
    for (long long j = k; j < issued; ++j)
      mbar_wait_bounded(&full[j % kRopeStages], static_cast<uint32_t>((j / kRopeStages) & 1), nullptr, nullptr, 0,
                        a.timeout_cycles / 4 + 1);
    bulk_wait_group_all();   // every store written before the CTA exits
  }
}

// float32 vectors: the first ceil(pairs / 2) float4 words of each 128-float vector.
__global__ void __launch_bounds__(256) rope_shift_f32_kernel(const RowRuns runs, const RopeTable tab) {
  const long long total = runs.start[runs.n];
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  const int words = (tab.pairs + 1) / 2;
  int seg = 0;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
    while (i >= runs.start[seg + 1]) ++seg;
    while (i < runs.start[seg]) --seg;
    float4* v = reinterpret_cast<float4*>(static_cast<char*>(runs.ptr[seg]) + (i - runs.start[seg]) * (kHeadDim * 4));
    for (int w = 0; w < words; ++w) {
      float4 x = v[w];
      const int p0 = 2 * w, p1 = 2 * w + 1;
      const float a0 = x.x * tab.c[p0] - x.y * tab.s[p0], b0 = x.x * tab.s[p0] + x.y * tab.c[p0];
      x.x = a0;
      x.y = b0;
      if (p1 < tab.pairs) {
        const float a1 = x.z * tab.c[p1] - x.w * tab.s[p1], b1 = x.z * tab.s[p1] + x.w * tab.c[p1];
        x.z = a1;
        x.w = b1;
      }
      v[w] = x;
    }
  }
}

template <int NW>
cudaError_t launch_nw(const RowRuns& runs, const RopeTable& tab, unsigned* err, long long timeout_cycles,
                      cudaStream_t st) {
  constexpr size_t smem = rope_smem_bytes<NW>();
  static PerDevice cap;
  int grid_cap = 0;
  cudaError_t e = cap.get(&grid_cap, [](int dev, int* v) {
    cudaError_t r = cudaFuncSetAttribute(rope_shift_tma_kernel<NW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (r != cudaSuccess) return r;
    int sms = 0, per_sm = 0;
    r = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (r != cudaSuccess) return r;
    r = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, rope_shift_tma_kernel<NW>, kRopeThreads, smem);
    if (r != cudaSuccess) return r;
    *v = sms * (per_sm > 0 ? per_sm : 1);
    return cudaSuccess;
  });
  if (e != cudaSuccess) return e;
  RopeTmaArgs a;
  a.n = runs.n;
  a.tab = tab;
  a.err = err;
  a.timeout_cycles = timeout_cycles;
  a.tile_start[0] = 0;
  for (int r = 0; r < runs.n; ++r) {
    const long long rows = runs.start[r + 1] - runs.start[r];
    if (rows > 0x7fffffffLL) return cudaErrorInvalidValue;   // TMA row coordinates are int
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kHeadDim) * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(8 * NW), static_cast<cuuint32_t>(kRopeRows)};
    const CUresult cr = encode_tiled(&a.map[r], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, runs.ptr[r], dims, strides, box,
                                     CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE);
    if (cr != CUDA_SUCCESS) return cudaErrorInvalidValue;
    a.tile_start[r + 1] = a.tile_start[r] + (rows + kRopeRows - 1) / kRopeRows;
  }
  const long long ntiles = a.tile_start[runs.n];
  if (ntiles <= 0) return cudaSuccess;
  const int grid = static_cast<int>(ntiles < grid_cap ? ntiles : grid_cap);
  rope_shift_tma_kernel<NW><<<grid, kRopeThreads, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_rope_shift_f32(const RowRuns& runs, const RopeTable& tab, cudaStream_t st) {
  const long long total = runs.start[runs.n];
  if (total <= 0 || tab.pairs <= 0) return cudaSuccess;
  const long long want = (total + 255) / 256;
  const int grid = static_cast<int>(want < 4096 ? want : 4096);
  rope_shift_f32_kernel<<<grid, 256, 0, st>>>(runs, tab);
  return cudaGetLastError();
}

cudaError_t launch_rope_shift(const RowRuns& runs, const RopeTable& tab, unsigned* err, long long timeout_cycles,
                              cudaStream_t st) {
  const long long total = runs.start[runs.n];
  if (total <= 0 || tab.pairs <= 0) return cudaSuccess;
  switch ((tab.pairs + 3) / 4) {
    case 1: return launch_nw<1>(runs, tab, err, timeout_cycles, st);
    case 2: return launch_nw<2>(runs, tab, err, timeout_cycles, st);
    case 3: return launch_nw<3>(runs, tab, err, timeout_cycles, st);
    case 4: return launch_nw<4>(runs, tab, err, timeout_cycles, st);
    case 5: return launch_nw<5>(runs, tab, err, timeout_cycles, st);
    case 6: return launch_nw<6>(runs, tab, err, timeout_cycles, st);
    case 7: return launch_nw<7>(runs, tab, err, timeout_cycles, st);
    case 8: return launch_nw<8>(runs, tab, err, timeout_cycles, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace pf
