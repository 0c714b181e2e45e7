// gemm_pair.cuh — the Y / dX GEMM on CTA pairs (tcgen05 cta_group::2).
//
//     out[M, Nout] = Aop[M, Kred] · Bop[Nout, Kred]ᵀ  +  E[M, r] · F[Nout, r]ᵀ
//
// Forward  (B_MN = false): Aop = X, Bop = W (K-major), E = s·XA, F = B      -> Y
// Backward (B_MN = true) : Aop = dY, Bop[k, n] = W[n, k] (MN-major), E = s·dY·B,
//                          F[k, j] = A[j, k] (MN-major)                      -> dX
//
// The LoRA term is one extra K fill after the main loop — possible because the
// adapter product is bracketed skinny-first ("Unsloth vs PyTorch: The ONLY Video You
// Need to Understand the Difference", transcript 1:35-2:00), so the N×K matrix B·A is
// never formed.  This kernel takes a bf16 weight (and, for the LM-head cross-entropy,
// a bf16 head); quantized weights go to lora_gemm_q_kernel (gemm_q.cuh).
//
// A cluster of two CTAs computes a 256×256 tile.  Each CTA loads its own 128 rows of A
// and its own 128 rows of the B tile (no multicast); the even CTA ("leader") issues
// tcgen05.mma.cta_group::2 (M=256, N=256, K=16), which reads both CTAs' shared memory
// and accumulates into both CTAs' TMEM (each CTA holds its 128 rows × 256 fp32 columns,
// double-buffered).  Per CTA this halves the operand bytes per MMA compared with a
// 128×256 single-CTA tile.
//
// Synchronisation.  TMA completions of both CTAs count on the leader's `full` barrier;
// the leader's MMA commits arrive on both CTAs' `empty` / `tfull` barriers (CTA mask
// 0b11); both CTAs' epilogue warps arrive on the leader's `tempty` barriers through
// cluster addresses.  Every wait is bounded.
//
// Work units (UnitWalk, gemm_common.cuh): whole tiles, or under the stream-K schedule
// (plain store epilogue only) also pieces of tiles, whose fp32 accumulators go to slots
// that streamk_fixup_kernel adds up.
//
// Roles per CTA: warp 0 TMA producer, warp 1 MMA issuer (leader) and TMEM owner,
// warps 2-5 epilogue.
#pragma once

#include "gemm_common.cuh"

namespace lora {

template <bool B_MN>
struct PairCfg {
  static constexpr int BM = 256, BN = 256, BK = 128;  // pair tile, K per pipeline fill
  static constexpr int HM = 128, HN = 128;            // per-CTA halves of A rows / B rows
  static constexpr int STAGES = 3;
  static constexpr int ATOM = 64;                       // 128-byte swizzle atom width (bf16)
  static constexpr int A_BYTES = HM * BK * 2;           // 32 KB (two 64-wide K atoms)
  static constexpr int B_BYTES = HN * BK * 2;           // 32 KB
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int NUM_EPI_WARPS = 4;
  static constexpr int NUM_THREADS = 32 * (2 + NUM_EPI_WARPS);
  // The SwiGLU-backward epilogue reads the saved gate and up values and rewrites them (four
  // times the bytes of a plain store): two warps per TMEM lane quarter, each draining half
  // of the columns, keep twice the loads in flight.
  template <int EPI>
  static constexpr int epi_warps() { return EPI == EPI_SWIGLU_BWD ? 8 : NUM_EPI_WARPS; }
  template <int EPI>
  static constexpr int threads() { return 32 * (2 + epi_warps<EPI>()); }
  static constexpr int TMEM_COLS = 512;
  static constexpr int NUM_BARS = 2 * STAGES + 5;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 8 * NUM_BARS + 16;
  static_assert(STAGE_BYTES % 1024 == 0, "stages must keep the 1024-byte swizzle alignment");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

template <bool B_MN, int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairCfg<B_MN>::template threads<EPI>(), 1)
    lora_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                          const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmF,
                          const PairParams p) {
  griddep_enter();  // the previous kernel in the stream completed (see ptx.cuh)
  using C = PairCfg<B_MN>;
  constexpr int NEPI = C::template epi_warps<EPI>();
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* full = bars;                    // leader: TMA bytes of both CTAs landed
  uint64_t* empty = bars + C::STAGES;       // both: the pair MMA finished reading the stage
  uint64_t* tfull = bars + 2 * C::STAGES;   // both: accumulator ready for the epilogue
  uint64_t* tempty = tfull + 2;             // leader: both CTAs drained the accumulator
  uint64_t* drain = tempty + 2;             // leader: final commit before TMEM release
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  volatile uint32_t* never_flag = tmem_slot + 2;  // stays 0: drain waits ignore the abort

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  const int num_m = (p.M + C::BM - 1) / C::BM;
  const int num_n = (p.Nout + EpiTile<EPI>::COLS - 1) / EpiTile<EPI>::COLS;
  const int ntiles = num_m * num_n;
  const bool sk = EPI == EPI_STORE && p.sk_on != 0;  // only the plain store epilogue runs stream-K
  const int nkb = (p.Kred + C::BK - 1) / C::BK;
  const int n_ext = p.r > 0 ? 1 : 0;         // one fill holds the whole LoRA block (r <= 128)
  const int tile_fills = nkb + n_ext;        // fills per tile
  const int ext_atoms = p.r > 64 ? 2 : 1;   // 64-wide rank atoms actually loaded
  const WaitCtl wc{abort_flag, p.status, p.wait_ns};

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&tfull[a]), 1);
      mbar_init(smem_u32(&tempty[a]), 2 * NEPI);
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
    tmem_alloc_pair(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  __syncwarp();
  cluster_sync();  // both CTAs' barriers exist before any cross-CTA arrive or TMA
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long long fills = 0;
      bool ok = true;
      UnitWalk w(pair, npairs, ntiles, tile_fills, sk, p.sk_dp_tiles);
      Unit un;
      while (ok && w.next(un)) {
        int mb, nb;
        pair_tile_coords(un.t, num_m, num_n, p.group_m, mb, nb);
        const int arow = mb * C::BM + static_cast<int>(rank) * C::HM;  // this CTA's rows of A
        const int brow = pair_brow<EPI>(nb, rank, p);  // this CTA's rows of the B tile
        // checked build: the tile exists and starts inside the output (a CTA's half of a
        // ragged tile may lie wholly past M or N: its boxes are TMA zero fills)
        if (!lora_check(mb < num_m && nb < num_n && mb * C::BM < p.M && nb * EpiTile<EPI>::COLS < p.Nout, wc)) {
          ok = false;
          break;
        }
        for (int kb = un.f0; kb < un.f1; ++kb) {
          if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, wc)) { ok = false; break; }
          const bool ext = kb >= nkb;
          if (!lora_check(ext ? kb - nkb < n_ext : kb * C::BK < p.Kred, wc)) { ok = false; break; }
          const uint32_t sA = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t sB = sA + C::A_BYTES;
          const uint32_t full_l = mapa_shared(smem_u32(&full[stage]), 0);
          if (leader) {
            uint32_t per_cta;
            if (!ext) per_cta = C::A_BYTES + C::B_BYTES;
            else per_cta = ext_atoms * (C::A_BYTES / 2) + (B_MN ? C::B_BYTES : ext_atoms * (C::B_BYTES / 2));
            mbar_arrive_expect_tx(smem_u32(&full[stage]), 2 * per_cta);
          }
          // every box is 64 wide × 128 rows; a K-major operand takes one box per
          // 64-wide K atom, an MN-major one (backward weight) one box per 64-wide MN chunk
          if (!ext) {
            tma_load_2d_pair(sA, &tmA, full_l, kb * C::BK, arow);
            tma_load_2d_pair(sA + C::A_BYTES / 2, &tmA, full_l, kb * C::BK + C::ATOM, arow);
            if (!B_MN) {
              tma_load_2d_pair(sB, &tmB, full_l, kb * C::BK, brow);
              tma_load_2d_pair(sB + C::B_BYTES / 2, &tmB, full_l, kb * C::BK + C::ATOM, brow);
            } else {
              tma_load_2d_pair(sB, &tmB, full_l, brow, kb * C::BK);
              tma_load_2d_pair(sB + C::B_BYTES / 2, &tmB, full_l, brow + C::ATOM, kb * C::BK);
            }
          } else {
            int seg = 0;
            while (seg + 1 < p.nseg && nb >= p.seg_end_tile[seg]) ++seg;
            const int e0 = seg * p.e_seg_stride;  // this tile's columns of E
            for (int h = 0; h < ext_atoms; ++h)
              tma_load_2d_pair(sA + h * (C::A_BYTES / 2), &tmE, full_l, e0 + h * C::ATOM, arow);
            if (!B_MN) {
              // the SwiGLU forward's odd CTA reads F from x = -f_shift: its first f_shift
              // columns are the zero fill, so the gate half of E meets zeros
              const int fx = EPI == EPI_SWIGLU_FWD ? -static_cast<int>(rank) * p.f_shift : 0;
              for (int h = 0; h < ext_atoms; ++h)
                tma_load_2d_pair(sB + h * (C::B_BYTES / 2), &tmF, full_l, fx + h * C::ATOM, brow);
            } else {
              tma_load_2d_pair(sB, &tmF, full_l, brow, 0);
              tma_load_2d_pair(sB + C::B_BYTES / 2, &tmF, full_l, brow + C::ATOM, 0);
            }
          }
          ++fills;
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        // let this CTA's loads that are still in flight land before shared memory goes away
        const long long first = fills > C::STAGES ? fills - C::STAGES : 0;
        const WaitCtl drain_wc{never_flag, nullptr, p.wait_ns};
        for (long long f = first; f < fills; ++f) {
          const int s = static_cast<int>(f % C::STAGES);
          const uint32_t ph = static_cast<uint32_t>((f / C::STAGES) & 1);
          if (leader) mbar_wait(smem_u32(&full[s]), ph, drain_wc);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (leader && lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(C::BM, C::BN, false, B_MN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      UnitWalk w(pair, npairs, ntiles, tile_fills, sk, p.sk_dp_tiles);
      Unit un;
      while (ok && w.next(un)) {
        if (!mbar_wait<true>(smem_u32(&tempty[acc]), acc_phase ^ 1u, wc)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(acc * C::BN);
        for (int kb = un.f0; kb < un.f1; ++kb) {
          if (!mbar_wait(smem_u32(&full[stage]), phase, wc)) { ok = false; break; }
          tc_fence_after();
          const bool ext = kb >= nkb;
          const uint32_t sA = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t sB = sA + C::A_BYTES;
          const int nk = ext ? (p.r + 15) / 16 : C::BK / 16;
          for (int k = 0; k < nk; ++k) {
            // K step k: atom k/4, 32-byte column (k%4) inside the K-major atom; for the
            // MN-major operand 16 K rows (2 KB) further down its 128-row chunks
            const uint32_t koff = (k >> 2) * (C::A_BYTES / 2) + (k & 3) * 32;
            const uint64_t ad = sdesc_sw128(sA + koff, 16, 1024);
            const uint64_t bd = B_MN ? sdesc_sw128(sB + k * 2048, C::B_BYTES / 2, 1024) : sdesc_sw128(sB + koff, 16, 1024);
            tc_mma_bf16_pair(d, ad, bd, idesc, (kb > un.f0 || k > 0) ? 1u : 0u);
          }
          tc_commit_pair_mc(smem_u32(&empty[stage]), 0x3);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit_pair_mc(smem_u32(&tfull[acc]), 0x3);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      // every pair MMA issued so far must finish before TMEM is released
      tc_commit_pair(smem_u32(drain));
      const WaitCtl drain_wc{never_flag, nullptr, p.wait_ns};
      mbar_wait(smem_u32(drain), 0, drain_wc);
    }
  } else if (warp < 2 + NEPI) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int quarter = warp & 3;  // TMEM lane quarter this warp may access
    int acc = 0;
    uint32_t acc_phase = 0;
    UnitWalk w(pair, npairs, ntiles, tile_fills, sk, p.sk_dp_tiles);
    Unit un;
    while (w.next(un)) {
      int mb, nb;
      pair_tile_coords(un.t, num_m, num_n, p.group_m, mb, nb);
      if (!mbar_wait_warp(smem_u32(&tfull[acc]), acc_phase, wc)) break;
      tc_fence_after();
      const int row = mb * C::BM + static_cast<int>(rank) * C::HM + quarter * 32 + lane;
      const uint32_t tbase =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * C::BN);
      if constexpr (EPI == EPI_SWIGLU_FWD) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          const int col0 = nb * 128 + c * 32;
          if (col0 >= p.Nout) break;  // warp-uniform
          uint32_t g[32], u[32];
          tmem_ld_32x32b_x32(tbase + c * 32, g);
          tmem_ld_32x32b_x32(tbase + 128 + c * 32, u);
          tmem_ld_wait();
          if (row < p.M) epi_swiglu_fwd_chunk(p, g, u, row, col0);
        }
      } else if constexpr (EPI == EPI_SWIGLU_BWD) {
        // with 8 epilogue warps, warps 2-5 and 6-9 split the 8 column chunks
        const int half = (warp - 2) >> 2;
        epi_swiglu_bwd_row(p, tbase, row, nb * C::BN, NEPI == 8 ? 4 * half : 0, NEPI == 8 ? 4 * half + 4 : 8);
      } else if constexpr (EPI == EPI_STORE) {
#pragma unroll 1
        for (int c = 0; c < C::BN / 32; ++c) {
          const int col0 = nb * C::BN + c * 32;
          if (col0 >= p.Nout) break;  // warp-uniform
          uint32_t v[32];
          tmem_ld_32x32b_x32(tbase + c * 32, v);
          tmem_ld_wait();
          if (row < p.M) {
            if (un.slot >= 0) epi_slot_chunk<C::BM>(p, v, un.slot, row - mb * C::BM, c * 32);
            else epi_store_chunk(p, v, row, col0);
          }
        }
      } else if constexpr (EPI == EPI_CE_LSE) {
        float m = -INFINITY, sum = 0.0f;
        const int y = row < p.M ? p.labels[row] : p.ignore_index;
        const int ylocal = (y == p.ignore_index) ? -1 : y - p.v0 - nb * C::BN;  // column in this tile
#pragma unroll 1
        for (int c = 0; c < C::BN / 32; ++c) {
          const int col0 = nb * C::BN + c * 32;
          if (col0 >= p.Nout) break;  // warp-uniform
          uint32_t v[32];
          tmem_ld_32x32b_x32(tbase + c * 32, v);
          tmem_ld_wait();
          const int nv = min(32, p.Nout - col0);
          float cm = -INFINITY;
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < nv) cm = fmaxf(cm, __uint_as_float(v[j]));
          const float nm = fmaxf(m, cm);
          float cs = 0.0f;
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < nv) cs += __expf(__uint_as_float(v[j]) - nm);
          sum = (m == -INFINITY ? 0.0f : sum * __expf(m - nm)) + cs;
          m = nm;
          if (ylocal >= c * 32 && ylocal < c * 32 + nv) {
            float z = 0.0f;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j == ylocal - c * 32) z = __uint_as_float(v[j]);
            p.label_logit[row] = z;
          }
        }
        if (row < p.M) {
          float2* part = reinterpret_cast<float2*>(p.lse_part) + static_cast<size_t>(nb) * p.M + row;
          *part = make_float2(m, sum);
        }
      } else if constexpr (EPI == EPI_CE_DLOGITS) {
        __nv_bfloat16* orow = p.out + static_cast<size_t>(row) * p.Nout;
        int ylocal = -1;
        float l = 0.0f, g = 0.0f;
        if (row < p.M) {
          const int y = p.labels[row];
          if (y != p.ignore_index) {
            ylocal = y - p.v0 - nb * C::BN;
            l = p.lse[row];
            g = p.dloss[row];
          }
        }
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
                uint32_t o[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int j0 = q * 8 + 2 * e;
                  const float d0 = g * (__expf(__uint_as_float(v[j0]) - l) - (c * 32 + j0 == ylocal ? 1.0f : 0.0f));
                  const float d1 =
                      g * (__expf(__uint_as_float(v[j0 + 1]) - l) - (c * 32 + j0 + 1 == ylocal ? 1.0f : 0.0f));
                  o[e] = pack_bf16x2(d0, d1);
                }
                *reinterpret_cast<uint4*>(orow + col0 + q * 8) = make_uint4(o[0], o[1], o[2], o[3]);
              }
            }
          }
        }
      } else if constexpr (EPI == EPI_ACC_F32) {
        float* arow = p.acc32 + static_cast<size_t>(row) * p.Nout;
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
                float f[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(v[q * 8 + e]);
                if (p.acc_mode & 1) {
                  const float4 a0 = *reinterpret_cast<const float4*>(arow + col0 + q * 8);
                  const float4 a1 = *reinterpret_cast<const float4*>(arow + col0 + q * 8 + 4);
                  f[0] += a0.x; f[1] += a0.y; f[2] += a0.z; f[3] += a0.w;
                  f[4] += a1.x; f[5] += a1.y; f[6] += a1.z; f[7] += a1.w;
                }
                if (p.acc_mode & 2) {
                  *reinterpret_cast<uint4*>(orow + col0 + q * 8) = make_uint4(
                      pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
                } else {
                  *reinterpret_cast<float4*>(arow + col0 + q * 8) = make_float4(f[0], f[1], f[2], f[3]);
                  *reinterpret_cast<float4*>(arow + col0 + q * 8 + 4) = make_float4(f[4], f[5], f[6], f[7]);
                }
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  __syncwarp();
  cluster_sync();  // the peer's TMEM and shared memory stay valid until the pair is done
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace lora
