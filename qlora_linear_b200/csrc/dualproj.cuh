// dualproj.cuh — one pass over dY for both rank-r products of the backward that read it:
//
//   T = dY·B       T[m][j] = Σ_c dY[m][c]·B[c][j]      (row projection, then s·T feeds the dX GEMM)
//   D = dYᵀ·XA     D[c][j] = Σ_m dY[m][c]·XA[m][j]     (column projection, s·D is dB)
//
// The hand-derived backward of "Unsloth vs PyTorch: The ONLY Video You Need to Understand
// the Difference" (transcript 0:43-2:00) takes both from the same dY; computed separately
// each one streams all of dY from HBM, here dY is read once.
//
// Work split: the CTA grid tiles dY into blocks of (row_tiles × 64) rows by (col_tiles × 256)
// columns.  A producer warp streams the block column tile by column tile, each column tile
// top to bottom, as 64 × 256 tiles (four 64 × 64 TMA boxes, 128-byte swizzle) together with
// the matching 64 × r rows of XA (32-byte swizzle); the 256 × r rows of B for the current
// column tile come in once per column tile and stay in registers as MMA fragments while the
// column tile streams by.  Four consumer warps contract every tile on the legacy warp MMA
// (these products are bandwidth-bound; shared-memory reads per tile are kept to the two
// fragment loads of dY, the XA tile and the T read-modify-write):
//   T rows of the tile   -> added into a shared-memory fp32 accumulator for the block's rows
//   D columns of the tile -> register accumulators, written once per column tile
// Each block writes fp32 partials, T for its column block and D for its row block; the
// finalize kernels add them in split order, so results do not depend on scheduling.
//
// The same stream serves the two passes over X, one product each (MODE):
//   DP_ROWS  T = X·Aᵀ      (the forward's XA; Q read from A [r][K] as stored)
//   DP_COLS  D = Xᵀ·R      (dA = (s·dY·B)ᵀ·X, computed as Xᵀ·(s·dY·B) and finalized transposed)
#pragma once

#include "ptx.cuh"

namespace lora {

constexpr int DP_TR = 64;                                 // dY rows per tile
constexpr int DP_TC = 256;                                // dY columns per tile (four TMA boxes)
constexpr int DP_RPAD = 16;                               // rank r = 8 or 16, padded to 16
constexpr int DP_STAGES = 3;
constexpr int DP_THREADS = 160;                           // 4 consumer warps + 1 producer warp
constexpr int DP_BOX_BYTES = DP_TR * 64 * 2;              // one 64 × 64 bf16 box (8 KB)
constexpr int DP_P_BYTES = DP_TR * DP_TC * 2;             // 32 KB
constexpr int DP_R_BYTES = DP_TR * DP_RPAD * 2;           // 2 KB
constexpr int DP_STAGE_BYTES = DP_P_BYTES + DP_R_BYTES;   // a multiple of 1024: boxes stay swizzle-aligned
constexpr int DP_Q_BYTES = DP_TC * DP_RPAD * 2;           // 8 KB of B per column tile
constexpr int DP_TPITCH = DP_RPAD + 8;                    // fp32 words per T accumulator row (conflict-free float2)
constexpr int DP_MAX_ROW_TILES = 16;                      // the T accumulator of 16 × 64 rows fills the rest
static_assert(DP_STAGE_BYTES % 1024 == 0, "stage size must keep the 128-byte swizzle atoms aligned");

enum : int { DP_BOTH = 0, DP_ROWS = 1, DP_COLS = 2 };

constexpr int dual_smem_bytes() {
  return 1024 + DP_STAGES * DP_STAGE_BYTES + 2 * DP_Q_BYTES + DP_MAX_ROW_TILES * DP_TR * DP_TPITCH * 4;
}

struct DualParams {
  float* partT;  // [gridDim.y][M][r]: T summed over this column block
  float* partD;  // [gridDim.x][C][r]: D summed over this row block
  int M, C, r;
  int row_tiles, col_tiles;  // tiles per block
  uint32_t* status;
  uint64_t wait_ns;
};

// tmP: dY block [M rows][C columns] (row pitch of dY), box 64 × 64, 128-byte swizzle.
// tmQ: B [C rows][r], box 16 × 256 (DP_ROWS: A [r rows][C], box 256 × 16).  tmR: XA
// [M rows][r] (row pitch of XA), box 16 × 64, 32-byte swizzle (16-byte chunk index ^= bit
// 2 of the row: conflict-free ldmatrix).  A mode that skips a product never touches its
// operand's map or its partials.
template <int MODE>
__global__ void __launch_bounds__(DP_THREADS, 1)
    dualproj_kernel(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmQ,
                    const __grid_constant__ CUtensorMap tmR, const DualParams p) {
  griddep_enter();  // the previous kernel in the stream completed (see ptx.cuh)
  constexpr bool DO_T = MODE != DP_COLS, DO_D = MODE != DP_ROWS;
  constexpr int STAGE_TX = DP_P_BYTES + (DO_D ? DP_R_BYTES : 0);
  extern __shared__ uint8_t dp_raw[];
  __shared__ __align__(8) uint64_t full[DP_STAGES], empty[DP_STAGES], qfull[2], qempty[2];
  __shared__ uint32_t abort_s, never_s;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dp_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + DP_STAGES * DP_STAGE_BYTES;
  float* tacc_s = reinterpret_cast<float*>(smem + DP_STAGES * DP_STAGE_BYTES + 2 * DP_Q_BYTES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntr = (p.M + DP_TR - 1) / DP_TR, ntc = (p.C + DP_TC - 1) / DP_TC;
  const int rt0 = blockIdx.x * p.row_tiles, ct0 = blockIdx.y * p.col_tiles;
  const int nrt = min(ntr, rt0 + p.row_tiles) - rt0;
  const int nct = min(ntc, ct0 + p.col_tiles) - ct0;
  const WaitCtl wc{&abort_s, p.status, p.wait_ns};

  if (threadIdx.x == 0) {
    for (int s = 0; s < DP_STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 4);
    }
    for (int q = 0; q < 2; ++q) {
      mbar_init(smem_u32(&qfull[q]), 1);
      mbar_init(smem_u32(&qempty[q]), 4);
    }
    abort_s = 0;
    never_s = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmP);
    if (DO_T) tma_prefetch_desc(&tmQ);
    if (DO_D) tma_prefetch_desc(&tmR);
  }
  if (DO_T)
    for (int i = threadIdx.x; i < max(nrt, 0) * DP_TR * DP_TPITCH; i += DP_THREADS) tacc_s[i] = 0.f;
  __syncthreads();
  if (nrt <= 0 || nct <= 0) return;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      long long fills = 0;
      int qloads = 0;
      bool ok = true;
      for (int ci = 0; ci < nct && ok; ++ci) {
        if (DO_T) {
          const int qb = ci & 1;
          if (ci >= 2 && !mbar_wait(smem_u32(&qempty[qb]), static_cast<uint32_t>(((ci >> 1) - 1) & 1), wc)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(smem_u32(&qfull[qb]), DP_Q_BYTES);
          if (MODE == DP_ROWS) tma_load_2d(sQ + qb * DP_Q_BYTES, &tmQ, smem_u32(&qfull[qb]), (ct0 + ci) * DP_TC, 0);
          else tma_load_2d(sQ + qb * DP_Q_BYTES, &tmQ, smem_u32(&qfull[qb]), 0, (ct0 + ci) * DP_TC);
          ++qloads;
        }
        for (int ri = 0; ri < nrt; ++ri) {
          const int s = static_cast<int>(fills % DP_STAGES);
          const uint32_t ph = static_cast<uint32_t>((fills / DP_STAGES) & 1);
          if (fills >= DP_STAGES && !mbar_wait(smem_u32(&empty[s]), ph ^ 1u, wc)) {
            ok = false;
            break;
          }
          const uint32_t st = sbase + s * DP_STAGE_BYTES;
          const uint32_t bar = smem_u32(&full[s]);
          const int y = (rt0 + ri) * DP_TR;
          // checked build: the tile's first row and column exist
          if (!lora_check(y < p.M && (ct0 + ci) * DP_TC < p.C, wc)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar, STAGE_TX);
#pragma unroll
          for (int b = 0; b < DP_TC / 64; ++b) tma_load_2d(st + b * DP_BOX_BYTES, &tmP, bar, (ct0 + ci) * DP_TC + b * 64, y);
          if (DO_D) tma_load_2d(st + DP_P_BYTES, &tmR, bar, 0, y);
          ++fills;
        }
      }
      if (!ok) {
        // loads still in flight must land before shared memory goes away
        const WaitCtl drain_wc{&never_s, nullptr, p.wait_ns};
        for (long long f = fills > DP_STAGES ? fills - DP_STAGES : 0; f < fills; ++f)
          mbar_wait(smem_u32(&full[f % DP_STAGES]), static_cast<uint32_t>((f / DP_STAGES) & 1), drain_wc);
        for (int q = qloads > 2 ? qloads - 2 : 0; q < qloads; ++q)
          mbar_wait(smem_u32(&qfull[q & 1]), static_cast<uint32_t>((q >> 1) & 1), drain_wc);
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers (warps 0-3)
  const int w = warp;
  long long fills = 0;
  bool ok = true;
  float* outD = p.partD + static_cast<size_t>(blockIdx.x) * p.C * p.r;
  for (int ci = 0; ci < nct && ok; ++ci) {
    // B (or Aᵀ) of this column tile as the MMA's second operand, 16 k-steps of 16 columns
    uint32_t qf[DP_TC / 16][4];
    if (DO_T) {
      const int qb = ci & 1;
      if (!mbar_wait_warp(smem_u32(&qfull[qb]), static_cast<uint32_t>((ci >> 1) & 1), wc)) {
        ok = false;
        break;
      }
      const uint32_t qa = sQ + qb * DP_Q_BYTES;
#pragma unroll
      for (int kk = 0; kk < DP_TC / 16; ++kk) {
        if (MODE == DP_ROWS) {
          // A [16 ranks][256 columns] as stored: rank j's row holds the k values, the
          // fragment layout of the MMA's second operand without a transpose
          const int j = (lane & 7) + ((lane >> 4) & 1) * 8;
          const int kc = kk * 16 + ((lane >> 3) & 1) * 8;
          ldsm_x4(qa + (j * DP_TC + kc) * 2, qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
        } else {
          const int kr = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
          const int jc = ((lane >> 4) & 1) * 8;
          ldsm_x4_t(qa + (kr * DP_RPAD + jc) * 2, qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
        }
      }
      // the next TMA load into this buffer (async proxy) must follow these ordinary
      // shared-memory reads: without the proxy fence it can overwrite them first
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&qempty[qb]));
    }
    float dacc[4][2][4];
#pragma unroll
    for (int f = 0; f < 4; ++f)
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) dacc[f][t][e] = 0.f;

    for (int ri = 0; ri < nrt; ++ri) {
      const int s = static_cast<int>(fills % DP_STAGES);
      if (!mbar_wait_warp(smem_u32(&full[s]), static_cast<uint32_t>((fills / DP_STAGES) & 1), wc)) {
        ok = false;
        break;
      }
      const uint32_t pa = sbase + s * DP_STAGE_BYTES;
      const uint32_t ra = pa + DP_P_BYTES;

      // T: rows 16w .. 16w+15 of the tile against all 256 columns
      float tacc[2][4];
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) tacc[t][e] = 0.f;
#pragma unroll
      for (int kk = 0; kk < (DO_T ? DP_TC / 16 : 0); ++kk) {
        const int row = w * 16 + (lane & 15);
        const int chunk = ((kk & 3) << 1) | (lane >> 4);
        uint32_t a0, a1, a2, a3;
        ldsm_x4(pa + (kk >> 2) * DP_BOX_BYTES + row * 128 + ((chunk ^ (row & 7)) << 4), a0, a1, a2, a3);
        mma_bf16_16816(tacc[0], a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
        mma_bf16_16816(tacc[1], a0, a1, a2, a3, qf[kk][2], qf[kk][3]);
      }
      // D: columns 64w .. 64w+63 (TMA box w) against all 64 rows
#pragma unroll
      for (int kk = 0; kk < (DO_D ? DP_TR / 16 : 0); ++kk) {
        const int mr = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int jchunk = (lane >> 4) & 1;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(ra + mr * (DP_RPAD * 2) + ((jchunk ^ ((mr >> 2) & 1)) << 4), b0, b1, b2, b3);
        const int ar = kk * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
#pragma unroll
        for (int f = 0; f < 4; ++f) {
          const int chunk = f * 2 + ((lane >> 3) & 1);
          uint32_t a0, a1, a2, a3;
          ldsm_x4_t(pa + w * DP_BOX_BYTES + ar * 128 + ((chunk ^ (ar & 7)) << 4), a0, a1, a2, a3);
          mma_bf16_16816(dacc[f][0], a0, a1, a2, a3, b0, b1);
          mma_bf16_16816(dacc[f][1], a0, a1, a2, a3, b2, b3);
        }
      }
      fence_proxy_async_smem();  // as for the B buffer: reads of the stage before its next TMA load
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
      ++fills;

      // this warp owns rows 16w .. 16w+15 of every tile of the block
      float* trow = tacc_s + (ri * DP_TR + w * 16 + (lane >> 2)) * DP_TPITCH + (lane & 3) * 2;
#pragma unroll
      for (int t = 0; t < (DO_T ? 2 : 0); ++t) {
        float2* lo = reinterpret_cast<float2*>(trow + t * 8);
        float2* hi = reinterpret_cast<float2*>(trow + 8 * DP_TPITCH + t * 8);
        float2 v = *lo;
        v.x += tacc[t][0];
        v.y += tacc[t][1];
        *lo = v;
        v = *hi;
        v.x += tacc[t][2];
        v.y += tacc[t][3];
        *hi = v;
      }
    }
    if (!ok) break;

    // D over this block's rows for the warp's 64 columns
#pragma unroll
    for (int f = 0; f < (DO_D ? 4 : 0); ++f) {
      const int c = (ct0 + ci) * DP_TC + w * 64 + f * 16 + (lane >> 2);
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int j = t * 8 + (lane & 3) * 2;
        if (t * 8 < p.r) {
          if (c < p.C)
            *reinterpret_cast<float2*>(outD + static_cast<size_t>(c) * p.r + j) = make_float2(dacc[f][t][0], dacc[f][t][1]);
          if (c + 8 < p.C)
            *reinterpret_cast<float2*>(outD + static_cast<size_t>(c + 8) * p.r + j) =
                make_float2(dacc[f][t][2], dacc[f][t][3]);
        }
      }
    }
  }
  if (!ok || !DO_T) return;

  // T over this block's columns for the warp's rows
  __syncwarp();
  float* outT = p.partT + static_cast<size_t>(blockIdx.y) * p.M * p.r;
  const int half = p.r / 2;  // float2 per row
  for (int ri = 0; ri < nrt; ++ri) {
    for (int i = lane; i < 16 * half; i += 32) {
      const int rr = i / half, jj = (i - rr * half) * 2;
      const int m = (rt0 + ri) * DP_TR + w * 16 + rr;
      if (m < p.M)
        *reinterpret_cast<float2*>(outT + static_cast<size_t>(m) * p.r + jj) =
            *reinterpret_cast<const float2*>(tacc_s + (ri * DP_TR + w * 16 + rr) * DP_TPITCH + jj);
    }
  }
}

}  // namespace lora
