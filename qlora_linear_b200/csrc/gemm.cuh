// gemm.cuh — persistent, warp-specialised tcgen05 GEMM with the LoRA term fused as one
// extra K block:
//
//     out[M, Nout] = Aop[M, Kred] · Bop[Nout, Kred]ᵀ  +  E[M, r] · F[Nout, r]ᵀ
//
// Forward  (B_MN = false): Aop = X, Bop = W (K-major), E = s·XA, F = B      -> Y
// Backward (B_MN = true) : Aop = dY, Bop[k, n] = W[n, k] (MN-major), E = s·dY·B,
//                          F[k, j] = A[j, k] (MN-major)                      -> dX
//
// The skinny-first bracketing ("Unsloth vs PyTorch: The ONLY Video You Need to
// Understand the Difference", transcript 1:35-2:00) is what makes the LoRA term a
// single K block of length r: the N×K product B·A is never formed.
//
// With W4 the frozen weight arrives as 4-bit codes ("Rev vs unsloth", fused
// quantized-LoRA paragraph): TMA brings the packed codes into shared memory and four
// dequant warps expand them, one 64-element scale block at a time, into the 128B-
// swizzled bf16 tile the tensor core reads.  The dequantized weight never reaches HBM.
//
// Tile 128×256×64, 1-CTA tcgen05.mma (M=128, N=256, K=16), fp32 accumulators in TMEM,
// double-buffered (2×256 columns) so the epilogue of one tile overlaps the main loop of
// the next.  Roles: warp 0 TMA producer, warp 1 MMA issuer (+ TMEM owner), warps 2-5
// epilogue, warps 6-9 dequant (W4 only).
#pragma once

#include "ptx.cuh"

namespace lora {

struct GemmParams {
  int M;           // rows of Aop / out
  int Nout;        // columns of out
  int Kred;        // reduction length (K forward, N backward)
  int r;           // adapter rank: ceil(r/64) extra K blocks; 0 = none
  __nv_bfloat16* out;  // [M, Nout] row-major
  uint32_t* status;    // device status word
  uint64_t wait_ns;    // bound of every mbarrier wait
  // 4-bit weight only
  const __half* absmax;  // [Nw*Kw/64]
  const float* codebook; // [16]
  int Nw, Kw;            // logical weight shape [Nw, Kw]
};

template <bool B_MN, bool W4>
struct GemmCfg {
  static constexpr int BM = 128, BN = 256, BK = 64;
  static constexpr int STAGES = W4 ? 3 : 4;
  static constexpr int A_BYTES = BM * BK * 2;               // 16 KB
  static constexpr int B_BYTES = BN * BK * 2;               // 32 KB
  static constexpr int C_BYTES = W4 ? BN * BK / 2 : 0;      // packed codes, 8 KB
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + C_BYTES;
  static constexpr int NUM_EPI_WARPS = 4;
  static constexpr int NUM_DEQ_WARPS = W4 ? 4 : 0;
  static constexpr int NUM_THREADS = 32 * (2 + NUM_EPI_WARPS + NUM_DEQ_WARPS);
  static constexpr int TMEM_COLS = 512;
  static constexpr int BAR_BYTES = 8 * (3 * STAGES + 4 + 1) + 16;
  static constexpr int SMEM_BYTES = 1024 /*align slack*/ + STAGES * STAGE_BYTES + BAR_BYTES;
  static constexpr int GROUP_M = 16;  // m-blocks per raster group (L2 reuse of W tiles)
};

__device__ __forceinline__ void tile_coords(int t, int num_m, int num_n, int group_m, int& mb, int& nb) {
  const int per_group = group_m * num_n;
  const int g = t / per_group;
  const int first_m = g * group_m;
  const int gm = min(group_m, num_m - first_m);
  const int within = t - first_m * num_n;
  mb = first_m + within % gm;
  nb = within / gm;
}

// Expand 8 codes (one 32-bit word) of one 64-element scale block into 8 bf16 using
// the block's 16 dequantized levels held as byte planes (lo bytes in L0..L3, hi bytes
// in H0..H3, entry e in byte e%4 of register e/4).  Element 2j sits in the low
// nibble of byte j, so the low 16 bits of `w` are the selectors of elements 0..3.
#ifndef LORA_EXPAND8_DEFINED
#define LORA_EXPAND8_DEFINED
__device__ __forceinline__ uint4 expand8(uint32_t w, const uint32_t (&L)[4], const uint32_t (&H)[4]) {
  uint4 o;
  {
    const uint32_t sel = w & 0x7777u;
    const uint32_t sel2 = ((w >> 1) & 0x4444u) | 0x3210u;
    const uint32_t lo = prmt(prmt(L[0], L[1], sel), prmt(L[2], L[3], sel), sel2);
    const uint32_t hi = prmt(prmt(H[0], H[1], sel), prmt(H[2], H[3], sel), sel2);
    o.x = prmt(lo, hi, 0x5140u);
    o.y = prmt(lo, hi, 0x7362u);
  }
  {
    const uint32_t w2 = w >> 16;
    const uint32_t sel = w2 & 0x7777u;
    const uint32_t sel2 = ((w2 >> 1) & 0x4444u) | 0x3210u;
    const uint32_t lo = prmt(prmt(L[0], L[1], sel), prmt(L[2], L[3], sel), sel2);
    const uint32_t hi = prmt(prmt(H[0], H[1], sel), prmt(H[2], H[3], sel), sel2);
    o.z = prmt(lo, hi, 0x5140u);
    o.w = prmt(lo, hi, 0x7362u);
  }
  return o;
}

// The 16 levels of one scale block, each bf16_rn(fp32_rn(codebook[c] * scale)), as
// byte planes for expand8().  The multiply is __fmul_rn so it is never fused.
__device__ __forceinline__ void block_levels(const float (&cb)[16], float scale, uint32_t (&L)[4], uint32_t (&H)[4]) {
  uint32_t v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = pack_bf16x2(__fmul_rn(cb[2 * i], scale), __fmul_rn(cb[2 * i + 1], scale));
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    L[i] = prmt(v[2 * i], v[2 * i + 1], 0x6420u);
    H[i] = prmt(v[2 * i], v[2 * i + 1], 0x7531u);
  }
}
#endif

template <bool B_MN, bool W4>
__global__ void __launch_bounds__(GemmCfg<B_MN, W4>::NUM_THREADS, 1)
    lora_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmF,
                     const GemmParams p) {
  using C = GemmCfg<B_MN, W4>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* full = bars;                      // TMA landed (A + B or codes)
  uint64_t* empty = bars + C::STAGES;         // MMA finished reading the stage
  uint64_t* deq = bars + 2 * C::STAGES;       // dequant wrote the bf16 weight tile (W4)
  uint64_t* tfull = bars + 3 * C::STAGES;     // accumulator ready for the epilogue
  uint64_t* tempty = tfull + 2;               // epilogue drained the accumulator
  uint64_t* drain = tempty + 2;               // final commit before TMEM release
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  volatile uint32_t* never_flag = tmem_slot + 2;  // stays 0: drain waits ignore the abort

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_m = (p.M + C::BM - 1) / C::BM;
  const int num_n = (p.Nout + C::BN - 1) / C::BN;
  const int ntiles = num_m * num_n;
  const int nkb = (p.Kred + C::BK - 1) / C::BK;
  const int n_ext = (p.r + 63) / 64;  // LoRA K blocks (64 ranks each)
  WaitCtl wc{abort_flag, p.status, p.wait_ns};

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
      mbar_init(smem_u32(&deq[s]), 32 * C::NUM_DEQ_WARPS > 0 ? 32 * C::NUM_DEQ_WARPS : 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&tfull[a]), 1);
      mbar_init(smem_u32(&tempty[a]), C::NUM_EPI_WARPS);
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    *never_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmE);
    tma_prefetch_desc(&tmF);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long long fills = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        int mb, nb;
        tile_coords(t, num_m, num_n, C::GROUP_M, mb, nb);
        for (int kb = 0; kb < nkb + n_ext; ++kb) {
          if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, wc)) { ok = false; break; }
          const bool ext = kb >= nkb;
          const int e = kb - nkb;
          uint8_t* sA = stage_base + stage * C::STAGE_BYTES;
          uint8_t* sB = sA + C::A_BYTES;
          uint8_t* sC = sB + C::B_BYTES;
          const uint32_t fb = smem_u32(&full[stage]);
          const uint32_t bbytes = (W4 && !ext) ? C::C_BYTES : C::B_BYTES;
          mbar_arrive_expect_tx(fb, C::A_BYTES + bbytes);
          if (!ext) {
            tma_load_2d(smem_u32(sA), &tmA, fb, kb * C::BK, mb * C::BM);
            if (W4) {
              if (!B_MN) tma_load_2d(smem_u32(sC), &tmB, fb, kb * (C::BK / 2), nb * C::BN);
              else tma_load_2d(smem_u32(sC), &tmB, fb, nb * (C::BN / 2), kb * C::BK);
            } else if (!B_MN) {
              tma_load_2d(smem_u32(sB), &tmB, fb, kb * C::BK, nb * C::BN);
            } else {
#pragma unroll
              for (int c = 0; c < C::BN / 64; ++c)
                tma_load_2d(smem_u32(sB + c * 8192), &tmB, fb, nb * C::BN + c * 64, kb * C::BK);
            }
          } else {
            tma_load_2d(smem_u32(sA), &tmE, fb, e * 64, mb * C::BM);
            if (!B_MN) {
              tma_load_2d(smem_u32(sB), &tmF, fb, e * 64, nb * C::BN);
            } else {
#pragma unroll
              for (int c = 0; c < C::BN / 64; ++c)
                tma_load_2d(smem_u32(sB + c * 8192), &tmF, fb, nb * C::BN + c * 64, e * 64);
            }
          }
          ++fills;
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        // let the loads already in flight land before the CTA's shared memory goes away
        const long long first = fills > C::STAGES ? fills - C::STAGES : 0;
        const WaitCtl drain_wc{never_flag, nullptr, p.wait_ns};
        for (long long f = first; f < fills; ++f) {
          const int s = static_cast<int>(f % C::STAGES);
          const uint32_t ph = static_cast<uint32_t>((f / C::STAGES) & 1);
          mbar_wait(smem_u32(&full[s]), ph, drain_wc);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(C::BM, C::BN, false, B_MN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        if (!mbar_wait(smem_u32(&tempty[acc]), acc_phase ^ 1u, wc)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(acc * C::BN);
        for (int kb = 0; kb < nkb + n_ext; ++kb) {
          if (!mbar_wait(smem_u32(&full[stage]), phase, wc)) { ok = false; break; }
          if (W4 && !mbar_wait(smem_u32(&deq[stage]), phase, wc)) { ok = false; break; }
          tc_fence_after();
          const bool ext = kb >= nkb;
          const uint32_t sA = smem_u32(stage_base + stage * C::STAGE_BYTES);
          const uint32_t sB = sA + C::A_BYTES;
          const int nk = ext ? min(C::BK / 16, (p.r - (kb - nkb) * 64 + 15) / 16) : C::BK / 16;
          for (int k = 0; k < nk; ++k) {
            const uint64_t ad = sdesc_sw128(sA + k * 32, 16, 1024);
            const uint64_t bd = B_MN ? sdesc_sw128(sB + k * 2048, 8192, 1024) : sdesc_sw128(sB + k * 32, 16, 1024);
            tc_mma_bf16(d, ad, bd, idesc, (kb > 0 || k > 0) ? 1u : 0u);
          }
          tc_commit(smem_u32(&empty[stage]));
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(smem_u32(&tfull[acc]));
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      // every MMA issued so far must finish before TMEM is released
      tc_commit(smem_u32(drain));
      const WaitCtl drain_wc{never_flag, nullptr, p.wait_ns};
      mbar_wait(smem_u32(drain), 0, drain_wc);
    }
  } else if (warp < 2 + C::NUM_EPI_WARPS) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lane quarter this warp may access
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
      int mb, nb;
      tile_coords(t, num_m, num_n, C::GROUP_M, mb, nb);
      if (!mbar_wait_warp(smem_u32(&tfull[acc]), acc_phase, wc)) break;
      tc_fence_after();
      const int row = mb * C::BM + quarter * 32 + lane;
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * C::BN);
      __nv_bfloat16* orow = p.out + static_cast<size_t>(row) * p.Nout;
#pragma unroll 1
      for (int c = 0; c < C::BN / 32; ++c) {
        const int col0 = nb * C::BN + c * 32;
        if (col0 >= p.Nout) break;  // warp-uniform
        uint32_t v[32];
        tmem_ld_32x32b_x32(tbase + c * 32, v);
        tmem_ld_wait();
        if (row < p.M) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (col0 + q * 8 < p.Nout) {
              uint4 o;
              o.x = pack_bf16x2(__uint_as_float(v[q * 8 + 0]), __uint_as_float(v[q * 8 + 1]));
              o.y = pack_bf16x2(__uint_as_float(v[q * 8 + 2]), __uint_as_float(v[q * 8 + 3]));
              o.z = pack_bf16x2(__uint_as_float(v[q * 8 + 4]), __uint_as_float(v[q * 8 + 5]));
              o.w = pack_bf16x2(__uint_as_float(v[q * 8 + 6]), __uint_as_float(v[q * 8 + 7]));
              *reinterpret_cast<uint4*>(orow + col0 + q * 8) = o;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&tempty[acc]));
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  } else if (W4) {
    // ------------------------------------------------------------ dequant (W4)
    const int dt = threadIdx.x - 32 * (2 + C::NUM_EPI_WARPS);  // 0..127
    float cb[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) cb[i] = __ldg(p.codebook + i);
    const int kblocks_w = p.Kw / 64;  // scale blocks per weight row
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
      int mb, nb;
      tile_coords(t, num_m, num_n, C::GROUP_M, mb, nb);
      for (int kb = 0; kb < nkb + n_ext; ++kb) {
        if (!mbar_wait(smem_u32(&full[stage]), phase, wc)) { ok = false; break; }
        if (kb < nkb) {
          uint8_t* sB = stage_base + stage * C::STAGE_BYTES + C::A_BYTES;
          const uint8_t* sC = sB + C::B_BYTES;
          if (!B_MN) {
            // tile: 256 weight rows n × 64 k; this thread: rows dt and dt+128
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int nl = dt + h * 128;
              const int n = nb * C::BN + nl;
              const float sc = n < p.Nw ? __half2float(p.absmax[static_cast<size_t>(n) * kblocks_w + kb]) : 0.f;
              uint32_t L[4], H[4];
              block_levels(cb, sc, L, H);
              const uint4 c0 = *reinterpret_cast<const uint4*>(sC + nl * 32);
              const uint4 c1 = *reinterpret_cast<const uint4*>(sC + nl * 32 + 16);
              const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
              uint8_t* rowp = sB + nl * 128;
#pragma unroll
              for (int u = 0; u < 8; ++u)
                *reinterpret_cast<uint4*>(rowp + ((u ^ (nl & 7)) << 4)) = expand8(cw[u], L, H);
            }
          } else {
            // tile: 64 weight rows n (reduction) × 256 k (output); this thread: row dt&63,
            // output half dt>>6 (two 64-wide scale blocks)
            const int nl = dt & 63;
            const int hh = dt >> 6;
            const int n = kb * C::BK + nl;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const int cchunk = hh * 2 + j;                  // 64-wide output chunk in the tile
              const int kblk = nb * (C::BN / 64) + cchunk;    // scale block along the weight row
              const float sc = (n < p.Nw && kblk < kblocks_w)
                                   ? __half2float(p.absmax[static_cast<size_t>(n) * kblocks_w + kblk])
                                   : 0.f;
              uint32_t L[4], H[4];
              block_levels(cb, sc, L, H);
              const uint8_t* crow = sC + nl * 128 + cchunk * 32;
              const uint4 c0 = *reinterpret_cast<const uint4*>(crow);
              const uint4 c1 = *reinterpret_cast<const uint4*>(crow + 16);
              const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
              uint8_t* rowp = sB + cchunk * 8192 + nl * 128;
#pragma unroll
              for (int u = 0; u < 8; ++u)
                *reinterpret_cast<uint4*>(rowp + ((u ^ (nl & 7)) << 4)) = expand8(cw[u], L, H);
            }
          }
          fence_proxy_async_smem();
        }
        mbar_arrive(smem_u32(&deq[stage]));
        if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace lora
