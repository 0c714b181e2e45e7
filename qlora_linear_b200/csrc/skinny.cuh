// skinny.cuh — the rank-r side products of the layer.  Each one streams a large
// activation (X or dY) once from HBM and contracts it with a skinny operand, so they
// are bandwidth-bound: the legacy warp MMA (m16n8k16, bf16 in, fp32 out) has plenty
// of throughput for r <= 128 and keeps these kernels simple.
//
//   rowproj:  part[s][m][j] = Σ_{k in split s} P[m][k] · Q(k, j)
//             XA  = X·Aᵀ   (Q = A, stored [r][K])       dY·B (Q = B, stored [N][r])
//   colproj:  part[s][c][j] = Σ_{m in split s} P[m][c] · R[m][j]
//             dB ∝ dYᵀ·XA  (P = dY, R = XA)             dA ∝ (dY·B)ᵀ·X as Xᵀ·(s·dY·B)
//
// Splits write fp32 partials; the finalize kernels add them in split order, so the
// result does not depend on scheduling ("warp-level reductions produce dA and dB",
// reduction order fixed).  The products follow the hand-derived backward of
// "Unsloth vs PyTorch: The ONLY Video You Need to Understand the Difference"
// (transcript 0:43-2:00) with the skinny-first bracketing.
#pragma once

#include "ptx.cuh"

namespace lora {

constexpr int SK_BM = 64;       // rows (rowproj) or output columns (colproj) per CTA
constexpr int SK_BK = 64;       // reduction step per stage
constexpr int SK_STAGES = 4;
constexpr int SK_THREADS = 128; // 4 warps × 16 rows
constexpr int SK_PITCH = 72;    // bf16 elements per smem row of a 64-wide tile (144 B: conflict-free ldmatrix)

template <int RPAD>
struct SkinnyCfg {
  static constexpr int QPITCH_T = RPAD + 8;  // pitch of a [64][RPAD] tile (odd number of 16 B chunks)
  static constexpr int P_ELEMS = SK_BM * SK_PITCH;
  static constexpr int QN_ELEMS = RPAD * SK_PITCH;    // Q stored [j][k]
  static constexpr int QT_ELEMS = SK_BK * QPITCH_T;   // Q or R stored [k][j]
};

template <int RPAD, bool Q_T>
constexpr int rowproj_smem_bytes() {
  return SK_STAGES * 2 * (SkinnyCfg<RPAD>::P_ELEMS + (Q_T ? SkinnyCfg<RPAD>::QT_ELEMS : SkinnyCfg<RPAD>::QN_ELEMS));
}
template <int RPAD>
constexpr int colproj_smem_bytes() {
  return SK_STAGES * 2 * (SkinnyCfg<RPAD>::P_ELEMS + SkinnyCfg<RPAD>::QT_ELEMS);
}

// One [rows × 64] bf16 tile of a row-major matrix into padded shared memory; rows >= nrows
// or columns >= ncols are zero-filled (ncols % 8 == 0).
__device__ __forceinline__ void load_tile_rows64(uint32_t sdst, int pitch, const __nv_bfloat16* g, int ldg, int row0,
                                                 int nrows, int col0, int ncols, int rows) {
  const int chunks = rows * 8;
  for (int c = threadIdx.x; c < chunks; c += SK_THREADS) {
    const int rr = c >> 3, cc = c & 7;
    const int gr = row0 + rr, gc = col0 + cc * 8;
    const bool in = gr < nrows && gc < ncols;
    const __nv_bfloat16* src = in ? g + static_cast<size_t>(gr) * ldg + gc : g;
    cp_async_16(sdst + (rr * pitch + cc * 8) * 2, src, in ? 16u : 0u);
  }
}
// [64 rows × RPAD cols] tile of the first r columns of a row-major matrix with row pitch
// ldg (r % 8 == 0), zero-filled beyond nrows / r.
template <int RPAD>
__device__ __forceinline__ void load_tile_rpad(uint32_t sdst, const __nv_bfloat16* g, int ldg, int r, int row0,
                                               int nrows) {
  constexpr int CPR = RPAD / 8;  // 16-byte chunks per row
  for (int c = threadIdx.x; c < SK_BK * CPR; c += SK_THREADS) {
    const int rr = c / CPR, cc = c % CPR;
    const int gr = row0 + rr, gc = cc * 8;
    const bool in = gr < nrows && gc < r;
    const __nv_bfloat16* src = in ? g + static_cast<size_t>(gr) * ldg + gc : g;
    cp_async_16(sdst + (rr * SkinnyCfg<RPAD>::QPITCH_T + cc * 8) * 2, src, in ? 16u : 0u);
  }
}

// part[split][m][j] (fp32, row pitch r) over k-tiles [kt0, kt1) of split blockIdx.y.
template <int RPAD, bool Q_T>
__global__ void __launch_bounds__(SK_THREADS)
    rowproj_kernel(const __nv_bfloat16* __restrict__ P, int ldp, const __nv_bfloat16* __restrict__ Q,
                   float* __restrict__ part, int M, int Kred, int r, int ktiles_per_split) {
  griddep_enter();  // the previous kernel in the stream completed (see ptx.cuh)
  using S = SkinnyCfg<RPAD>;
  constexpr int QE = Q_T ? S::QT_ELEMS : S::QN_ELEMS;
  extern __shared__ __align__(16) uint8_t sk_smem[];
  const uint32_t sbase = smem_u32(sk_smem);
  auto sP = [&](int st) { return sbase + st * (S::P_ELEMS + QE) * 2; };
  auto sQ = [&](int st) { return sP(st) + S::P_ELEMS * 2; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * SK_BM;
  const int ktiles = (Kred + SK_BK - 1) / SK_BK;
  const int kt0 = blockIdx.y * ktiles_per_split;
  const int kt1 = min(ktiles, kt0 + ktiles_per_split);
  const int nt = kt1 - kt0;

  auto issue = [&](int i) {
    const int st = i % SK_STAGES;
    const int k0 = (kt0 + i) * SK_BK;
    load_tile_rows64(sP(st), SK_PITCH, P, ldp, m0, M, k0, Kred, SK_BM);
    if (Q_T) {
      // Q stored [Kred][r]: rows k0..k0+63
      load_tile_rpad<RPAD>(sQ(st), Q, r, r, k0, Kred);
    } else {
      // Q stored [r][Kred]: RPAD rows j, columns k0..k0+63
      load_tile_rows64(sQ(st), SK_PITCH, Q, Kred, 0, r, k0, Kred, RPAD);
    }
  };

  float acc[RPAD / 8][4];
#pragma unroll
  for (int t = 0; t < RPAD / 8; ++t)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[t][q] = 0.f;

#pragma unroll
  for (int i = 0; i < SK_STAGES - 1; ++i) {
    if (i < nt) issue(i);
    cp_async_commit();
  }
  for (int i = 0; i < nt; ++i) {
    cp_async_wait<SK_STAGES - 2>();
    __syncthreads();
    if (i + SK_STAGES - 1 < nt) issue(i + SK_STAGES - 1);
    cp_async_commit();
    const int st = i % SK_STAGES;
    const uint32_t pa = sP(st), qa = sQ(st);
#pragma unroll
    for (int kk = 0; kk < SK_BK / 16; ++kk) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(pa + ((warp * 16 + (lane & 15)) * SK_PITCH + kk * 16 + (lane >> 4) * 8) * 2, a0, a1, a2, a3);
#pragma unroll
      for (int jp = 0; jp < RPAD / 16; ++jp) {
        uint32_t b0, b1, b2, b3;
        if (Q_T) {
          const int kr = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
          const int jc = jp * 16 + ((lane >> 4) & 1) * 8;
          ldsm_x4_t(qa + (kr * S::QPITCH_T + jc) * 2, b0, b1, b2, b3);
        } else {
          const int jr = jp * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
          const int kc = kk * 16 + ((lane >> 3) & 1) * 8;
          ldsm_x4(qa + (jr * SK_PITCH + kc) * 2, b0, b1, b2, b3);
        }
        mma_bf16_16816(acc[2 * jp], a0, a1, a2, a3, b0, b1);
        mma_bf16_16816(acc[2 * jp + 1], a0, a1, a2, a3, b2, b3);
      }
    }
  }
  cp_async_wait<0>();

  float* out = part + static_cast<size_t>(blockIdx.y) * M * r;
  const int row = m0 + warp * 16 + (lane >> 2);
#pragma unroll
  for (int t = 0; t < RPAD / 8; ++t) {
    const int col = t * 8 + (lane & 3) * 2;
    if (t * 8 < r) {
      if (row < M) *reinterpret_cast<float2*>(out + static_cast<size_t>(row) * r + col) = make_float2(acc[t][0], acc[t][1]);
      if (row + 8 < M)
        *reinterpret_cast<float2*>(out + static_cast<size_t>(row + 8) * r + col) = make_float2(acc[t][2], acc[t][3]);
    }
  }
}

// part[split][c][j] (fp32, row pitch r) = Σ over m-tiles [mt0, mt1) of P[m][c]·R[m][j].
template <int RPAD>
__global__ void __launch_bounds__(SK_THREADS)
    colproj_kernel(const __nv_bfloat16* __restrict__ P, int ldp, const __nv_bfloat16* __restrict__ R, int ldr,
                   float* __restrict__ part, int M, int Kout, int r, int mtiles_per_split) {
  griddep_enter();  // the previous kernel in the stream completed (see ptx.cuh)
  using S = SkinnyCfg<RPAD>;
  extern __shared__ __align__(16) uint8_t sk_smem[];
  const uint32_t sbase = smem_u32(sk_smem);
  auto sP = [&](int st) { return sbase + st * (S::P_ELEMS + S::QT_ELEMS) * 2; };
  auto sR = [&](int st) { return sP(st) + S::P_ELEMS * 2; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c0 = blockIdx.x * SK_BM;
  const int mtiles = (M + SK_BK - 1) / SK_BK;
  const int mt0 = blockIdx.y * mtiles_per_split;
  const int mt1 = min(mtiles, mt0 + mtiles_per_split);
  const int nt = mt1 - mt0;

  auto issue = [&](int i) {
    const int st = i % SK_STAGES;
    const int mrow = (mt0 + i) * SK_BK;
    load_tile_rows64(sP(st), SK_PITCH, P, ldp, mrow, M, c0, Kout, SK_BK);
    load_tile_rpad<RPAD>(sR(st), R, ldr, r, mrow, M);
  };

  float acc[RPAD / 8][4];
#pragma unroll
  for (int t = 0; t < RPAD / 8; ++t)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[t][q] = 0.f;

#pragma unroll
  for (int i = 0; i < SK_STAGES - 1; ++i) {
    if (i < nt) issue(i);
    cp_async_commit();
  }
  for (int i = 0; i < nt; ++i) {
    cp_async_wait<SK_STAGES - 2>();
    __syncthreads();
    if (i + SK_STAGES - 1 < nt) issue(i + SK_STAGES - 1);
    cp_async_commit();
    const int st = i % SK_STAGES;
    const uint32_t pa = sP(st), ra = sR(st);
#pragma unroll
    for (int kk = 0; kk < SK_BK / 16; ++kk) {
      // A(row = c, col = m) = P[m][c]: transposed load of the [m][c] tile
      uint32_t a0, a1, a2, a3;
      {
        const int mr = kk * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
        const int cc = warp * 16 + ((lane >> 3) & 1) * 8;
        ldsm_x4_t(pa + (mr * SK_PITCH + cc) * 2, a0, a1, a2, a3);
      }
#pragma unroll
      for (int jp = 0; jp < RPAD / 16; ++jp) {
        uint32_t b0, b1, b2, b3;
        const int mr = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int jc = jp * 16 + ((lane >> 4) & 1) * 8;
        ldsm_x4_t(ra + (mr * S::QPITCH_T + jc) * 2, b0, b1, b2, b3);
        mma_bf16_16816(acc[2 * jp], a0, a1, a2, a3, b0, b1);
        mma_bf16_16816(acc[2 * jp + 1], a0, a1, a2, a3, b2, b3);
      }
    }
  }
  cp_async_wait<0>();

  float* out = part + static_cast<size_t>(blockIdx.y) * Kout * r;
  const int row = c0 + warp * 16 + (lane >> 2);
#pragma unroll
  for (int t = 0; t < RPAD / 8; ++t) {
    const int col = t * 8 + (lane & 3) * 2;
    if (t * 8 < r) {
      if (row < Kout)
        *reinterpret_cast<float2*>(out + static_cast<size_t>(row) * r + col) = make_float2(acc[t][0], acc[t][1]);
      if (row + 8 < Kout)
        *reinterpret_cast<float2*>(out + static_cast<size_t>(row + 8) * r + col) = make_float2(acc[t][2], acc[t][3]);
    }
  }
}

// out1 = bf16(Σ_s part[s]), out2 = bf16(scale · Σ_s part[s]); either may be null.
// part is [splits][rows][r]; summed in split order.  Row i of the result goes to
// out[i*opitch .. i*opitch + r) (opitch >= r lets a result fill one column block of a
// wider matrix).
__global__ void finalize_rows_kernel(const float* __restrict__ part, int splits, size_t n, int r, int opitch,
                                     float scale, __nv_bfloat16* __restrict__ out1, __nv_bfloat16* __restrict__ out2) {
  griddep_enter();  // the previous kernel in the stream completed (see ptx.cuh)
  for (size_t i = (static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 2; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x * 2) {
    const size_t o = (opitch == r) ? i : (i / r) * opitch + i % r;
    float2 acc = *reinterpret_cast<const float2*>(part + i);
    for (int s = 1; s < splits; ++s) {
      const float2 v = *reinterpret_cast<const float2*>(part + static_cast<size_t>(s) * n + i);
      acc.x += v.x;
      acc.y += v.y;
    }
    if (out1) *reinterpret_cast<uint32_t*>(out1 + o) = pack_bf16x2(acc.x, acc.y);
    if (out2) *reinterpret_cast<uint32_t*>(out2 + o) = pack_bf16x2(scale * acc.x, scale * acc.y);
  }
}

// out = scale · Σ_s part[s] where part is [splits][C][r]; written as [C][r], or as [r][C]
// when transpose is set.  OutT = __nv_bfloat16 rounds to nearest even; OutT = float keeps
// the fp32 value (adapter gradients that are summed over data-parallel ranks first).
__device__ __forceinline__ void store_out(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
__device__ __forceinline__ void store_out(float* p, float v) { *p = v; }

template <typename OutT>
__global__ void finalize_cols_kernel(const float* __restrict__ part, int splits, int C, int r, float scale,
                                     int transpose, OutT* __restrict__ out) {
  griddep_enter();  // the previous kernel in the stream completed (see ptx.cuh)
  const size_t n = static_cast<size_t>(C) * r;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    // with transpose, i enumerates the output [r][C] so writes are coalesced
    size_t src;
    if (transpose) {
      const size_t j = i / C, c = i % C;
      src = c * r + j;
    } else {
      src = i;
    }
    float acc = part[src];
    for (int s = 1; s < splits; ++s) acc += part[static_cast<size_t>(s) * n + src];
    store_out(out + i, scale * acc);
  }
}

// dst = bf16_rn(src), n elements (the fp32 adapter gradients after their sum over ranks).
__global__ void round_bf16_kernel(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst, size_t n) {
  griddep_enter();  // the previous kernel in the stream completed (see ptx.cuh)
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    dst[i] = __float2bfloat16_rn(src[i]);
}

}  // namespace lora
