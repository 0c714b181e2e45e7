// tcproj.cuh — the rank-r side products for ranks above 16 on the tensor cores
// (tcgen05, one CTA, accumulator in TMEM), fed by TMA:
//
//   row projection     part[s][m][j] = Σ_{c in split s} P[m][c] · Q(c, j)
//        TP_ROWS_K   Q(c, j) = A[j][c]   (X·Aᵀ, A stored [r][K]: the MMA's B operand K-major)
//        TP_ROWS_MN  Q(c, j) = B[c][j]   (dY·B, B stored [N][r]: the B operand MN-major)
//   column projection  part[s][c][j] = Σ_{m in split s} P[m][c] · R[m][j]
//        TP_COLS     dB ∝ dYᵀ·XA (P = dY, R = XA); dA ∝ (dY·B)ᵀ·X as Xᵀ·(s·dY·B) (P = X)
//
// These are the skinny-first products of the hand-derived backward ("Unsloth vs PyTorch:
// The ONLY Video You Need to Understand the Difference", transcript 0:43-2:00).  Each
// streams a large activation (X or dY) once; at rank r it does r multiply-adds per
// element read, which for r = 64 or 128 is more than the legacy warp MMA keeps up with at
// the HBM rate, so here the tensor core runs them: M = 128 output rows (row projection)
// or 128 output columns (column projection), N = the rank padded to 64 or 128 (TMA fills
// the padding with zeros), K = 16 per MMA, 64 per pipeline fill.
//
// One P tile per fill serves either way: [128 rows × 64 columns] read K-major for the
// row projection, or [64 rows × 128 columns] (two 64 × 64 boxes) read MN-major for the
// column projection (the output columns are the MMA's M dimension).  Q / R tiles are
// [rpad × 64] K-major (TP_ROWS_K) or [64 × rpad] MN-major in 64-wide chunks.  All tiles
// use the 128-byte swizzle.
//
// Work unit = one CTA: output tile `t` (128 rows or columns) and split `s` of the
// reduction (fills [s·fps, (s+1)·fps)); partials are fp32 [splits][rows][r] and the
// finalize kernels add them in split order, so results do not depend on scheduling.
// Warps: 0 TMA producer, 1 MMA issuer and TMEM owner, 2-5 epilogue.  Every wait is
// bounded.
#pragma once

#include "ptx.cuh"

namespace lora {

constexpr int TP_BM = 128;                       // output rows (or columns) per tile
constexpr int TP_BK = 64;                        // reduction per fill
constexpr int TP_STAGES = 3;
constexpr int TP_THREADS = 192;
constexpr int TP_P_BYTES = TP_BM * TP_BK * 2;    // 16 KB
constexpr int TP_Q_BYTES = 128 * TP_BK * 2;      // 16 KB (rank padded to at most 128)
constexpr int TP_STAGE_BYTES = TP_P_BYTES + TP_Q_BYTES;
constexpr int TP_TMEM_COLS = 128;

enum : int { TP_ROWS_K = 0, TP_ROWS_MN = 1, TP_COLS = 2 };

constexpr int tcproj_smem_bytes() { return 1024 + TP_STAGES * TP_STAGE_BYTES + 256; }

struct TcProjParams {
  float* part;          // [splits][rows][r]
  int rows;             // output rows: M (row projection) or C (column projection)
  int red;              // reduction length: C (row projection) or M (column projection)
  int r, rpad;          // rank and its padding (64 or 128)
  int splits, fps;      // splits of the reduction and fills per split
  uint32_t* status;
  uint64_t wait_ns;
};

// tmP: the activation P [M][C] (row pitch of P), box 64 × 128 (row projection) or 64 × 64
// (column projection), 128-byte swizzle.  tmQ: A [r][K] with box 64 × rpad (TP_ROWS_K),
// or B [N][r] / R [M][r] with box 64 × 64 (the other modes), 128-byte swizzle.
template <int MODE>
__global__ void __launch_bounds__(TP_THREADS, 1)
    tcproj_kernel(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmQ,
                  const TcProjParams p) {
  griddep_enter();  // the previous kernel in the stream completed (see ptx.cuh)
  extern __shared__ __align__(1024) uint8_t tp_raw[];
  __shared__ __align__(8) uint64_t full[TP_STAGES], empty[TP_STAGES], tfull;
  __shared__ uint32_t tmem_slot, abort_s, never_s;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tp_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x / p.splits, split = blockIdx.x % p.splits;
  const int nkb = (p.red + TP_BK - 1) / TP_BK;
  const int kb0 = split * p.fps;
  const int kb1 = min(nkb, kb0 + p.fps);
  const int row0 = tile * TP_BM;
  const int nq = p.rpad / 64;  // 64-wide rank chunks (MN-major Q / R)
  const WaitCtl wc{&abort_s, p.status, p.wait_ns};

  if (threadIdx.x == 0) {
    for (int s = 0; s < TP_STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(&tfull), 1);
    abort_s = 0;
    never_s = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmP);
    tma_prefetch_desc(&tmQ);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_slot), TP_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int fills = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb, ++fills) {
        const int s = fills % TP_STAGES;
        const uint32_t ph = static_cast<uint32_t>((fills / TP_STAGES) & 1);
        if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1u, wc)) { ok = false; break; }
        // checked build: the output tile and the fill's reduction slice exist
        if (!lora_check(row0 < p.rows && kb * TP_BK < p.red && split < p.splits, wc)) { ok = false; break; }
        const uint32_t sP = smem_u32(smem + s * TP_STAGE_BYTES);
        const uint32_t sQ = sP + TP_P_BYTES;
        const uint32_t bar = smem_u32(&full[s]);
        const uint32_t qbytes = MODE == TP_ROWS_K ? p.rpad * TP_BK * 2 : nq * 64 * 64 * 2;
        mbar_arrive_expect_tx(bar, TP_P_BYTES + qbytes);
        if (MODE == TP_COLS) {
          // 64 reduction rows × 128 output columns: two 64 × 64 boxes
          tma_load_2d(sP, &tmP, bar, row0, kb * TP_BK);
          tma_load_2d(sP + TP_P_BYTES / 2, &tmP, bar, row0 + 64, kb * TP_BK);
        } else {
          tma_load_2d(sP, &tmP, bar, kb * TP_BK, row0);  // 128 rows × 64 reduction columns
        }
        if (MODE == TP_ROWS_K) {
          tma_load_2d(sQ, &tmQ, bar, kb * TP_BK, 0);  // rpad ranks × 64 (ranks >= r: zeros)
        } else {
          for (int q = 0; q < nq; ++q) tma_load_2d(sQ + q * 8192, &tmQ, bar, q * 64, kb * TP_BK);
        }
      }
      if (!ok) {
        // loads still in flight land before shared memory goes away
        const WaitCtl drain_wc{&never_s, nullptr, p.wait_ns};
        for (int f = fills > TP_STAGES ? fills - TP_STAGES : 0; f < fills; ++f)
          mbar_wait(smem_u32(&full[f % TP_STAGES]), static_cast<uint32_t>((f / TP_STAGES) & 1), drain_wc);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(TP_BM, p.rpad, MODE == TP_COLS, MODE != TP_ROWS_K);
      int fills = 0;
      for (int kb = kb0; kb < kb1; ++kb, ++fills) {
        const int s = fills % TP_STAGES;
        if (!mbar_wait(smem_u32(&full[s]), static_cast<uint32_t>((fills / TP_STAGES) & 1), wc)) break;
        tc_fence_after();
        const uint32_t sP = smem_u32(smem + s * TP_STAGE_BYTES);
        const uint32_t sQ = sP + TP_P_BYTES;
#pragma unroll
        for (int k = 0; k < TP_BK / 16; ++k) {
          // K-major: 32 bytes further along the 128-byte rows; MN-major: 16 rows (2 KB)
          // further down, 64-wide chunks 8 KB apart
          const uint64_t ad = MODE == TP_COLS ? sdesc_sw128(sP + k * 2048, 8192, 1024) : sdesc_sw128(sP + k * 32, 16, 1024);
          const uint64_t bd = MODE == TP_ROWS_K ? sdesc_sw128(sQ + k * 32, 16, 1024) : sdesc_sw128(sQ + k * 2048, 8192, 1024);
          tc_mma_bf16(tmem_base, ad, bd, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
        }
        tc_commit(smem_u32(&empty[s]));
      }
      // the epilogue reads the accumulator once every MMA completed (also after an abort:
      // the commit tracks whatever was issued)
      tc_commit(smem_u32(&tfull));
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-5)
    const int quarter = warp & 3;
    const int lr = quarter * 32 + lane;  // tile row of this thread (TMEM lane)
    const int grow = row0 + lr;
    const WaitCtl ewc{&never_s, p.status, p.wait_ns};
    if (mbar_wait_warp(smem_u32(&tfull), 0, ewc) && !abort_s) {
      tc_fence_after();
      float* dst = p.part + (static_cast<size_t>(split) * p.rows + grow) * p.r;
      const bool any = kb1 > kb0;  // an empty split contributes zeros
#pragma unroll 1
      for (int c = 0; c < p.rpad / 32; ++c) {
        if (c * 32 >= p.r) break;  // warp-uniform
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + c * 32, v);
        tmem_ld_wait();
        if (grow < p.rows) {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            if (c * 32 + q * 4 < p.r)
              *reinterpret_cast<float4*>(dst + c * 32 + q * 4) =
                  any ? make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                    __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]))
                      : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TP_TMEM_COLS);
  }
}

}  // namespace lora
