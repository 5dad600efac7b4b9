// append_copy.cu -- moves a finished block's K/V and compressed Kc/Vc into
// the cache arena (PackForcing (arXiv), "Dual-Resolution Shifting
// Mechanism": the new full-resolution tokens replace the oldest recent
// ones, the compressed copy is kept for when the block ages into the mid
// partition).  All runs of one append go in a single launch; 16-byte
// vectors, four loads in flight per thread, grid = the CTAs resident at once.
#include "pf_internal.h"

namespace pf {

namespace {

__global__ void __launch_bounds__(256) copy_runs_kernel(const CopyRuns runs) {
  const long long total = runs.start[runs.n];
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  const long long first = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  int seg = 0;
  constexpr int U = 4;
  for (long long base = first; base < total; base += stride * U) {
    uint4 v[U];
    long long idx[U];
    int sg[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      idx[u] = base + u * stride;
      sg[u] = -1;
      if (idx[u] < total) {
        while (idx[u] >= runs.start[seg + 1]) ++seg;
        while (idx[u] < runs.start[seg]) --seg;
        sg[u] = seg;
        v[u] = static_cast<const uint4*>(runs.src[seg])[idx[u] - runs.start[seg]];
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (sg[u] >= 0) static_cast<uint4*>(runs.dst[sg[u]])[idx[u] - runs.start[sg[u]]] = v[u];
    }
  }
}

}  // namespace

cudaError_t launch_copy(const CopyRuns& runs, cudaStream_t st) {
  const long long total = runs.start[runs.n];
  if (total <= 0) return cudaSuccess;
  static PerDevice cap;
  int grid_cap = 0;
  cudaError_t e = cap.get(&grid_cap, [](int dev, int* v) { return one_wave_grid(copy_runs_kernel, dev, v); });
  if (e != cudaSuccess) return e;
  const long long want = (total + 1023) / 1024;
  const int grid = static_cast<int>(want < grid_cap ? want : grid_cap);
  copy_runs_kernel<<<grid, 256, 0, st>>>(runs);
  return cudaGetLastError();
}

}  // namespace pf
