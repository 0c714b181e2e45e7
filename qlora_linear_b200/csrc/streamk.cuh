// streamk.cuh — the second kernel of the GEMMs' stream-K schedule: adds the fp32 pieces of
// every output tile that the schedule cut (gemm_common.cuh, UnitWalk) and writes the bf16
// output.  HBM-bound: each cut tile's pieces are read once and its output written once.
#pragma once

#include "gemm_common.cuh"

namespace lora {

// Block (x, y) handles the tile in which the boundary between pairs x and x + 1 falls, if
// that boundary is the tile's first, rows [8y, 8y + 8) of it: thread (row, 8-column chunk).
// The pieces of a tile come from consecutive pairs; they are added in pair order, two
// loads in flight at a time.
template <int TILE_ROWS>
__global__ void __launch_bounds__(256) streamk_fixup_kernel(const float* __restrict__ kpart, __nv_bfloat16* __restrict__ out,
                                                            int M, int Nout, int num_m, int num_n, int group_m,
                                                            int dp_tiles, int ntiles, int L, int P) {
  griddep_enter();  // the previous kernel in the stream completed (see ptx.cuh)
  const int p = blockIdx.x + 1;
  const long long F = static_cast<long long>(ntiles - dp_tiles) * L;
  const long long b = static_cast<long long>(p) * F / P;
  if (b % L == 0) return;  // the boundary falls between two tiles
  const long long ts = (b / L) * L, te = ts + L;
  if (static_cast<long long>(p - 1) * F / P > ts) return;  // an earlier boundary lies in this tile
  int mb, nb;
  pair_tile_coords(dp_tiles + static_cast<int>(b / L), num_m, num_n, group_m, mb, nb);
  const int lr = blockIdx.y * 8 + (threadIdx.x >> 5), lc = (threadIdx.x & 31) * 8;
  const int row = mb * TILE_ROWS + lr, col = nb * 256 + lc;
  if (row >= M || col >= Nout) return;
  auto gq = [&](int q) { return static_cast<long long>(q) * F / P; };
  auto piece = [&](int q) {  // this thread's 8 values of pair q's piece of the tile
    const int slot = gq(q) >= ts ? 2 * q : 2 * q + 1;
    return reinterpret_cast<const float4*>(kpart + (static_cast<size_t>(slot) * TILE_ROWS + lr) * 256 + lc);
  };
  int qend = p;  // pairs p - 1 .. qend - 1 hold pieces of the tile
  while (qend < P && gq(qend) < te) ++qend;
  float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  int q = p - 1;
  for (; q + 1 < qend; q += 2) {
    const float4* s0 = piece(q);
    const float4* s1 = piece(q + 1);
    const float4 x0 = s0[0], y0 = s0[1], x1 = s1[0], y1 = s1[1];
    a[0] += x0.x; a[1] += x0.y; a[2] += x0.z; a[3] += x0.w;
    a[4] += y0.x; a[5] += y0.y; a[6] += y0.z; a[7] += y0.w;
    a[0] += x1.x; a[1] += x1.y; a[2] += x1.z; a[3] += x1.w;
    a[4] += y1.x; a[5] += y1.y; a[6] += y1.z; a[7] += y1.w;
  }
  if (q < qend) {
    const float4* s0 = piece(q);
    const float4 x0 = s0[0], y0 = s0[1];
    a[0] += x0.x; a[1] += x0.y; a[2] += x0.z; a[3] += x0.w;
    a[4] += y0.x; a[5] += y0.y; a[6] += y0.z; a[7] += y0.w;
  }
  *reinterpret_cast<uint4*>(out + static_cast<size_t>(row) * Nout + col) =
      make_uint4(pack_bf16x2(a[0], a[1]), pack_bf16x2(a[2], a[3]), pack_bf16x2(a[4], a[5]), pack_bf16x2(a[6], a[7]));
}

}  // namespace lora
