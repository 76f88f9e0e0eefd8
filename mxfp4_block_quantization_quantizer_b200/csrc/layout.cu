// Scale bytes in the blocked order of block-scaled tensor-core GEMMs.
//
// Source: "Oscillation-Reduced MXFP4 Training for Vision Transformers",
// abstract (MX is supported by the Blackwell architecture); the order is
// NVIDIA's published one-dimensional block-scaling-factor layout: tiles of
// 128 rows x 4 groups, 512 bytes each, along the groups first; inside a tile
// the 16-byte line i holds the 4 scales of rows i, i+32, i+64 and i+96.
//
// One thread writes one 16-byte line: four 4-byte pieces from four rows of
// the row-major scales (one 32-bit load each when every row starts 4-byte
// aligned), zero outside the matrix. Lines are consecutive across a warp, so
// the stores are fully coalesced; the input is 1/32 of the quantized tensor
// and is read once.
#include "launch.cuh"

namespace mxfp4 {

namespace {

constexpr int kLayoutThreads = 256;

template <bool VEC>
__global__ void __launch_bounds__(kLayoutThreads)
    k_scales_blocked(const uint8_t* __restrict__ s, int64_t rows,
                     int64_t groups, int64_t group_tiles, int64_t n_lines,
                     uint4* __restrict__ out) {
  const int64_t stride = int64_t(gridDim.x) * kLayoutThreads;
  for (int64_t line = int64_t(blockIdx.x) * kLayoutThreads + threadIdx.x;
       line < n_lines; line += stride) {
    const int64_t tile = line >> 5;
    const int i = int(line & 31);
    const int64_t r0 = (tile / group_tiles) * 128 + i;
    const int64_t g0 = (tile % group_tiles) * 4;
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int64_t r = r0 + 32 * k;
      w[k] = 0;
      if (r >= rows) continue;
      const uint8_t* p = s + r * groups + g0;
      if (VEC) {
        w[k] = *reinterpret_cast<const uint32_t*>(p);
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (g0 + j < groups) w[k] |= uint32_t(p[j]) << (8 * j);
      }
    }
    out[line] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

}  // namespace

cudaError_t launch_scales_blocked(const uint8_t* scales, int64_t rows,
                                  int64_t groups, uint8_t* blocked,
                                  cudaStream_t s) {
  const int64_t group_tiles = (groups + 3) / 4;
  const int64_t n_lines = ((rows + 127) / 128) * group_tiles * 32;
  const int64_t blocks = (n_lines + kLayoutThreads - 1) / kLayoutThreads;
  const bool vec = groups % 4 == 0 &&
                   (reinterpret_cast<uintptr_t>(scales) & 3u) == 0;
  uint4* out = reinterpret_cast<uint4*>(blocked);
  if (vec) {
    const int grid = persistent_grid(
        reinterpret_cast<const void*>(k_scales_blocked<true>), kLayoutThreads,
        0, blocks);
    k_scales_blocked<true><<<grid, kLayoutThreads, 0, s>>>(
        scales, rows, groups, group_tiles, n_lines, out);
  } else {
    const int grid = persistent_grid(
        reinterpret_cast<const void*>(k_scales_blocked<false>), kLayoutThreads,
        0, blocks);
    k_scales_blocked<false><<<grid, kLayoutThreads, 0, s>>>(
        scales, rows, groups, group_tiles, n_lines, out);
  }
  return cudaGetLastError();
}

}  // namespace mxfp4
