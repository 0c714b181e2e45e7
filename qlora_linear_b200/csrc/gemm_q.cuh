// gemm_q.cuh — the Y / dX GEMM for quantized frozen weights (4-bit blockwise codes,
// int8 or fp8 e4m3 with row scales) on CTA pairs, with 512-row pair tiles.
//
//     out[M, Nout] = Aop[M, Kred] · Bop[Nout, Kred]ᵀ  +  E[M, r] · F[Nout, r]ᵀ
//
// Same operation and operand roles as lora_gemm_pair_kernel (gemm_pair.cuh); the weight
// arrives as codes and is expanded to bf16 in shared memory by the CTA's dequant warps
// ("Rev vs unsloth", fused quantized-LoRA paragraph: the quantized weight is never
// dequantized to device memory).
//
// Why a separate kernel.  The expanded B tile is written by ordinary shared-memory
// stores, which compete with the tensor core's operand reads; measured per 128-deep
// fill of a 256×256 pair tile, the expansion and its proxy fence took about as long as
// the fill's MMAs, and the MMAs themselves ran a third slower.  Here every expanded B
// tile feeds two M = 256 MMAs (a 512-row pair tile with two accumulators), which halves
// the expanded bytes and the expansion work per MMA FLOP.  To keep three-plus stages
// within shared memory the fills are 64 deep (16 MMAs of M=256, N=256, K=16 each, the
// same MMA work per fill as the bf16 kernel's 128-deep fills), four stages, and the two
// accumulators fill all 512 TMEM columns: instead of double-buffering, each accumulator
// has its own full/empty barrier pair, so the next tile's MMAs into the first
// accumulator start while the epilogue still drains the second.
//
// Work units as in lora_gemm_pair_kernel (UnitWalk): whole tiles, and under the stream-K
// schedule pieces of tiles, a piece being any consecutive range of the tile's code fills
// and LoRA fills.
//
// Codes do not pass through shared memory.  Each dequant thread loads the 32 (4-bit) or
// 64 (8-bit) code bytes it expands, with its block scale, into registers two of its
// group's fills ahead, and writes the stage's B tile as soon as the MMAs of the stage's
// previous fill have completed (the `empty` barrier the producer waits for too).  With the
// codes in the stage's TMA load instead, every fill's expansion waited for a load issued
// only when the stage came free, and the four-stage ring spent ~1.5k more cycles per
// round trip than its fills' MMA time covers: two stages ran 37% slower than four, and
// the kernel ran ~10% slower than the same kernel with the expansion skipped.
//
// Roles per CTA (16 warps; warp w runs on sub-partition w % 4): warp 0 TMA producer,
// warp 1 MMA issuer (leader) and TMEM owner, warps 2-5 epilogue, warps 9 and 13 forward
// the dequant warps' completion of each fill to the leader (one per dequant group: the
// cluster-scope arrive holds its thread for ~1000 cycles), and warps 6-8, 10-12, 14-15
// dequantize.  No dequant warp shares the MMA warp's sub-partition:
// a tcgen05.mma whose issue waits for room in the tensor core's queue holds up the other
// warps of its sub-partition, and dequant warps placed there lagged their CTA's others
// by ~2400 cycles per fill in a timeline of the kernel (untraced: +5% on the QLoRA
// shape).  Every wait is bounded.
#pragma once

#include "dequant.cuh"
#include "gemm_common.cuh"

namespace lora {

template <bool B_MN, int WF>
struct QCfg {
  static constexpr bool W4 = WF == WF_BLOCK4;
  static constexpr int BM = 512, BN = 256, BK = 64;  // pair tile, K per pipeline fill
  static constexpr int MB = 2;                        // 256-row M blocks (accumulators) per pair tile
  static constexpr int HM = 128, HN = 128;            // per-CTA rows of an A block / of the B tile
  static constexpr int STAGES = 4;
  static constexpr int ATOM = 64;                       // 128-byte swizzle atom width (bf16)
  static constexpr int A_BLOCK_BYTES = HM * BK * 2;     // 16 KB
  static constexpr int A_BYTES = MB * A_BLOCK_BYTES;    // 32 KB
  static constexpr int B_BYTES = HN * BK * 2;           // 16 KB (two 8 KB MN atoms when B is MN-major)
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int CODE_WORDS = W4 ? 2 : 4;         // 16-byte code words a dequant thread expands per fill
  static constexpr int NUM_EPI_WARPS = 4;
  static constexpr int NUM_DEQ_WARPS = 8;
  static constexpr int NUM_THREADS = 32 * 16;
  static constexpr int FWD_WARP = 9;    // forwarder of dequant group 0
  static constexpr int FWD_WARP2 = 13;  // forwarder of dequant group 1
  // dequant warps 6,7,8,10,11,12,14,15 -> dequant index 0..7
  static __device__ __forceinline__ int deq_index(int warp) { return warp < 9 ? warp - 6 : (warp < 13 ? warp - 7 : warp - 8); }
  static constexpr int TMEM_COLS = 512;  // MB accumulators of BN fp32 columns
  static constexpr int NUM_BARS = 4 * STAGES + 2 * MB + 1;
  // Output staging of the store epilogue: two 32-row × 32-column bf16 buffers per epilogue
  // warp, 64-byte swizzle, written to global memory by TMA stores.
  static constexpr bool STAGED_STORE = true;
  static constexpr int STG_BYTES = 2048;
  static constexpr int NSTG = 2;  // staging buffers per epilogue warp (a power of two)
  static constexpr int EPI_STG_BYTES = STAGED_STORE ? NUM_EPI_WARPS * NSTG * STG_BYTES : 0;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + EPI_STG_BYTES + 8 * NUM_BARS + 16;
  static_assert(STAGE_BYTES % 1024 == 0, "stages must keep the 1024-byte swizzle alignment");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

template <bool B_MN, int WF, int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(QCfg<B_MN, WF>::NUM_THREADS, 1)
    lora_gemm_q_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmE,
                       const __grid_constant__ CUtensorMap tmF,
                       const __grid_constant__ CUtensorMap tmO, const PairParams p) {
  griddep_enter();  // the previous kernel in the stream completed (see ptx.cuh)
  using C = QCfg<B_MN, WF>;
  constexpr bool W4 = C::W4;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stg_base = smem + C::STAGES * C::STAGE_BYTES;  // epilogue staging (1024-aligned)
  uint64_t* bars = reinterpret_cast<uint64_t*>(stg_base + C::EPI_STG_BYTES);
  uint64_t* full = bars;                    // leader: TMA bytes of both CTAs landed
  uint64_t* empty = bars + C::STAGES;       // both: the pair MMA finished reading the stage
  uint64_t* deq = bars + 2 * C::STAGES;     // leader: both CTAs' expanded tiles written (one forward each)
  uint64_t* tfull = bars + 3 * C::STAGES;   // both: accumulator b ready for the epilogue
  uint64_t* tempty = tfull + C::MB;         // leader: both CTAs drained accumulator b
  uint64_t* drain = tempty + C::MB;         // leader: final commit before TMEM release
  uint64_t* deql = drain + 1;               // both: this CTA's dequant warps wrote the stage
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(deql + C::STAGES);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  volatile uint32_t* never_flag = tmem_slot + 2;

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
  const int n_ext = p.r > 0 ? (p.r + C::ATOM - 1) / C::ATOM : 0;  // 64 ranks per LoRA fill
  const int tile_fills = nkb + n_ext;  // fills per tile
  const WaitCtl wc{abort_flag, p.status, p.wait_ns};

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
      mbar_init(smem_u32(&deq[s]), 2);
      mbar_init(smem_u32(&deql[s]), C::NUM_DEQ_WARPS / 2);  // the stage's dequant group
    }
    for (int b = 0; b < C::MB; ++b) {
      mbar_init(smem_u32(&tfull[b]), 1);
      mbar_init(smem_u32(&tempty[b]), 2 * C::NUM_EPI_WARPS);
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    *never_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmE);
    tma_prefetch_desc(&tmF);
    if (EPI == EPI_STORE && C::STAGED_STORE) tma_prefetch_desc(&tmO);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  __syncwarp();
  cluster_sync();
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
        const int arow = mb * C::BM + static_cast<int>(rank) * C::HM;  // this CTA's rows of A block 0
        const int brow = pair_brow<EPI>(nb, rank, p);
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
          if (leader) mbar_arrive_expect_tx(smem_u32(&full[stage]), 2 * (C::A_BYTES + (ext ? C::B_BYTES : 0)));
          if (!ext) {
            for (int b = 0; b < C::MB; ++b)
              tma_load_2d_pair(sA + b * C::A_BLOCK_BYTES, &tmA, full_l, kb * C::BK, arow + b * 256);
          } else {
            const int e = kb - nkb;
            int seg = 0;
            while (seg + 1 < p.nseg && nb >= p.seg_end_tile[seg]) ++seg;
            const int e0 = seg * p.e_seg_stride + e * C::ATOM;  // this fill's columns of E
            for (int b = 0; b < C::MB; ++b)
              tma_load_2d_pair(sA + b * C::A_BLOCK_BYTES, &tmE, full_l, e0, arow + b * 256);
            if (!B_MN) {
              const int fx = EPI == EPI_SWIGLU_FWD ? -static_cast<int>(rank) * p.f_shift : 0;
              tma_load_2d_pair(sB, &tmF, full_l, fx + e * C::ATOM, brow);  // 64 ranks × 128 rows
            } else {
              tma_load_2d_pair(sB, &tmF, full_l, brow, e * C::ATOM);       // 64 columns × 64 ranks
              tma_load_2d_pair(sB + C::B_BYTES / 2, &tmF, full_l, brow + C::ATOM, e * C::ATOM);
            }
          }
          ++fills;
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
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
      constexpr uint32_t idesc = idesc_bf16_f32(256, C::BN, false, B_MN);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t tphase = 0;  // parity of the accumulator barriers for this tile
      bool ok = true;
      UnitWalk w(pair, npairs, ntiles, tile_fills, sk, p.sk_dp_tiles);
      Unit un;
      // the MMAs of one fill into accumulator b (the fill's first MMA overwrites it when the
      // fill is the unit's first)
      auto issue = [&](int st, int kb, int b, bool first_fill) {
        const bool ext = kb >= nkb;
        const uint32_t sA = smem_u32(smem + st * C::STAGE_BYTES);
        const uint32_t sB = sA + C::A_BYTES;
        const int nk = ext ? min(C::BK / 16, (p.r - (kb - nkb) * C::ATOM + 15) / 16) : C::BK / 16;
        const uint32_t d = tmem_base + static_cast<uint32_t>(b * C::BN);
        for (int k = 0; k < nk; ++k) {
          const uint64_t ad = sdesc_sw128(sA + b * C::A_BLOCK_BYTES + k * 32, 16, 1024);
          const uint64_t bd = B_MN ? sdesc_sw128(sB + k * 2048, C::B_BYTES / 2, 1024) : sdesc_sw128(sB + k * 32, 16, 1024);
          tc_mma_bf16_pair(d, ad, bd, idesc, (!first_fill || k > 0) ? 1u : 0u);
        }
      };
      auto ready = [&](int st, uint32_t ph) -> bool {  // the fill's tiles of both CTAs are in place
        if (!mbar_wait(smem_u32(&full[st]), ph, wc)) return false;
        if (!mbar_wait<true>(smem_u32(&deq[st]), ph, wc)) return false;
        tc_fence_after();
        return true;
      };
      auto advance = [](int& st, uint32_t& ph) {
        if (++st == C::STAGES) { st = 0; ph ^= 1u; }
      };
      // A unit's first and last fills (up to a stage ring's worth each) are issued one
      // accumulator at a time.  First fills: accumulator 0's MMAs of all of them start as
      // soon as the epilogue has drained accumulator 0 of the previous tile, while it still
      // drains accumulator 1.  Last fills: accumulator 0 is complete, and handed to the
      // epilogue, while accumulator 1's last MMAs still run.  Fills in between alternate the
      // accumulators fill by fill and release each stage at once.  Each accumulator sums its
      // fills in the same order either way.
      auto group = [&](int lo, int hi, bool first, bool last) -> bool {
        int st = stage;
        uint32_t ph = phase;
        if (first) {
          if (!mbar_wait<true>(smem_u32(&tempty[0]), tphase ^ 1u, wc)) return false;
          tc_fence_after();
        }
        for (int j = lo; j < hi; ++j) {
          if (!ready(st, ph)) return false;
          issue(st, un.f0 + j, 0, j == 0);
          advance(st, ph);
        }
        if (last) tc_commit_pair_mc(smem_u32(&tfull[0]), 0x3);
        if (first) {
          if (!mbar_wait<true>(smem_u32(&tempty[1]), tphase ^ 1u, wc)) return false;
          tc_fence_after();
        }
        for (int j = lo; j < hi; ++j) {
          issue(stage, un.f0 + j, 1, j == 0);
          tc_commit_pair_mc(smem_u32(&empty[stage]), 0x3);
          advance(stage, phase);
        }
        if (last) tc_commit_pair_mc(smem_u32(&tfull[1]), 0x3);
        return true;
      };
      static_assert(C::MB == 2, "the issue order is written for two accumulators");
      while (ok && w.next(un)) {
        const int n = un.f1 - un.f0;
        const int g0 = min(n, C::STAGES);          // first fills [0, g0)
        const int g1 = max(g0, n - C::STAGES);     // last fills [g1, n)
        if (!group(0, g0, true, g0 == n)) { ok = false; break; }
        for (int j = g0; j < g1; ++j) {
          if (!ready(stage, phase)) { ok = false; break; }
          issue(stage, un.f0 + j, 0, false);
          issue(stage, un.f0 + j, 1, false);
          tc_commit_pair_mc(smem_u32(&empty[stage]), 0x3);
          advance(stage, phase);
        }
        if (!ok) break;
        if (g1 < n && !group(g1, n, false, true)) { ok = false; break; }
        tphase ^= 1u;
      }
      tc_commit_pair(smem_u32(drain));
      const WaitCtl drain_wc{never_flag, nullptr, p.wait_ns};
      mbar_wait(smem_u32(drain), 0, drain_wc);
    }
  } else if (warp < 2 + C::NUM_EPI_WARPS) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int quarter = warp & 3;  // TMEM lane quarter this warp may access
    const uint32_t stg = smem_u32(stg_base) + static_cast<uint32_t>((warp - 2) * C::NSTG * C::STG_BYTES);
    int sb = 0;  // staging buffer of the next staged chunk
    uint32_t tphase = 0;
    bool ok = true;
    UnitWalk w(pair, npairs, ntiles, tile_fills, sk, p.sk_dp_tiles);
    Unit un;
    while (ok && w.next(un)) {
      int mb, nb;
      pair_tile_coords(un.t, num_m, num_n, p.group_m, mb, nb);
      for (int b = 0; b < C::MB; ++b) {
        if (!mbar_wait_warp(smem_u32(&tfull[b]), tphase, wc)) { ok = false; break; }
        tc_fence_after();
        const int row = mb * C::BM + b * 256 + static_cast<int>(rank) * C::HM + quarter * 32 + lane;
        const uint32_t tbase =
            tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(b * C::BN);
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
          epi_swiglu_bwd_row(p, tbase, row, nb * C::BN);
        } else if (C::STAGED_STORE && un.slot < 0) {
          // 32 rows × 32 columns per chunk through a staging buffer and one TMA store (rows
          // past M and columns past Nout are not written); chunk c + 1's TMEM load is in
          // flight while chunk c is converted and staged.  Lane i writes row i, 16-byte unit
          // u at position u ^ ((i >> 1) & 3), the 64-byte swizzle of the output map.
          const int row0 = row - lane;  // first of the warp's 32 rows
          const int nch = min(C::BN / 32, (p.Nout - nb * C::BN + 31) / 32);  // warp-uniform
          auto stage_chunk = [&](const uint32_t (&v)[32], int c) {
            const uint32_t buf = stg + static_cast<uint32_t>(sb * C::STG_BYTES);
            if (lane == 0) bulk_wait_read<C::NSTG - 1>();  // the store that last read this buffer
            __syncwarp();
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint32_t a = buf + lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4);
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a),
                           "r"(pack_bf16x2(__uint_as_float(v[8 * q + 0]), __uint_as_float(v[8 * q + 1]))),
                           "r"(pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3]))),
                           "r"(pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5]))),
                           "r"(pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7])))
                           : "memory");
            }
            fence_proxy_async_smem();  // the generic writes before the TMA store reads them
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmO, buf, nb * C::BN + c * 32, row0);
              bulk_commit();
            }
            sb = (sb + 1) & (C::NSTG - 1);
          };
          if (row0 < p.M && nch > 0) {
            uint32_t va[32], vb[32];
            tmem_ld_32x32b_x32(tbase, va);
            tmem_ld_wait();
#pragma unroll 1
            for (int c = 0; c < nch; c += 2) {
              if (c + 1 < nch) tmem_ld_32x32b_x32(tbase + (c + 1) * 32, vb);
              stage_chunk(va, c);
              if (c + 1 < nch) {
                tmem_ld_wait();
                if (c + 2 < nch) tmem_ld_32x32b_x32(tbase + (c + 2) * 32, va);
                stage_chunk(vb, c + 1);
                if (c + 2 < nch) tmem_ld_wait();
              }
            }
          }
        } else {
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
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[b]), 0));
      }
      tphase ^= 1u;
    }
  } else if (warp == C::FWD_WARP || warp == C::FWD_WARP2) {
    // ------------------------------------------------------------ forwarders (both CTAs)
    // The dequant warps signal a CTA-local barrier (release at CTA scope); these warps turn
    // each completed fill into the one cluster-scope release arrive the leader's MMA
    // issuer waits for, warp 9 for the stages of dequant group 0, warp 13 for group 1.  A
    // release at cluster scope costs about a fill's worth of cycles when every dequant
    // warp issues its own, and holds the forwarding thread for ~1000 cycles.
    const int fgrp = warp == C::FWD_WARP ? 0 : 1;
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      UnitWalk w(pair, npairs, ntiles, tile_fills, sk, p.sk_dp_tiles);
      Unit un;
      while (ok && w.next(un)) {
        for (int kb = un.f0; kb < un.f1; ++kb) {
          if ((stage & 1) == fgrp) {
            if (!mbar_wait(smem_u32(&deql[stage]), phase, wc)) { ok = false; break; }
            mbar_arrive_cluster(mapa_shared(smem_u32(&deq[stage]), 0));
          }
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ dequant (both CTAs)
    // Two groups of four warps take turns: group g expands the fills held in stages g and
    // g + 2 (an even number of stages, so every fill of a stage belongs to one group), and a
    // thread expands one whole 64-element scale block per fill, so each block's 16 levels
    // are built once:
    //   forward:  weight row `row` (0..127) of this CTA's B rows, the fill's 64-deep slice;
    //   backward: weight row `row` (0..63) of the fill, 64-column half `h` of this CTA's 128.
    static_assert(C::STAGES % 2 == 0, "stages alternate between the two dequant groups");
    constexpr int NW = C::CODE_WORDS;
    const int dq = C::deq_index(warp);   // 0..7
    const int grp = dq >> 2;             // 0 or 1
    const int gt = (dq & 3) * 32 + lane;  // 0..127 within the group
    const int row = !B_MN ? gt : (gt & 63);
    const int h = !B_MN ? 0 : (gt >> 6);
    float cb[16];
    if (W4) {
#pragma unroll
      for (int i = 0; i < 16; ++i) cb[i] = __ldg(p.codebook + i);
    }
    const long long kblocks_w = p.Kw / 64;  // 4-bit scale blocks per weight row
    const long long row_bytes = W4 ? p.Kw / 2 : p.Kw;
    // What this thread expands in one code fill: the scale as raw bits (a fp16 block scale
    // for 4-bit, a fp32 row scale for 8-bit; converted only where the fill uses it) and the
    // code bytes, the same bytes a TMA box of the fill would hold, zero outside the weight
    // (weight rows >= Nw, columns >= Kw: 16-byte words, Kw being a multiple of 16 codes).
    struct FillCodes {
      uint32_t s;
      uint4 c[NW];
    };
    auto fill_codes = [&](int t, int kb, FillCodes& q) {
      int mb, nb;
      pair_tile_coords(t, num_m, num_n, p.group_m, mb, nb);
      const int brow = pair_brow<EPI>(nb, rank, p);
      // forward: weight row brow + row, bytes of the fill's 64 columns; backward: weight
      // row kb·64 + row, bytes of this thread's 64 of the CTA's output columns
      const long long n = !B_MN ? static_cast<long long>(brow) + row : static_cast<long long>(kb) * C::BK + row;
      const long long x = !B_MN ? static_cast<long long>(kb) * (NW * 16)
                                : static_cast<long long>(W4 ? brow / 2 : brow) + h * (NW * 16);
      const bool in_rows = n < p.Nw;
      const uint4* src = reinterpret_cast<const uint4*>(p.codes + (in_rows ? n : 0) * row_bytes + x);
#pragma unroll
      for (int i = 0; i < NW; ++i)
        q.c[i] = in_rows && x + i * 16 < row_bytes ? __ldg(src + i) : make_uint4(0u, 0u, 0u, 0u);
      q.s = 0u;
      if (in_rows) {
        if (W4) {
          const long long kblk = !B_MN ? kb : (brow + h * 64) / 64;
          if (kblk < kblocks_w)
            q.s = static_cast<uint32_t>(__ldg(reinterpret_cast<const unsigned short*>(p.absmax) + n * kblocks_w + kblk));
        } else {
          q.s = __float_as_uint(__ldg(p.row_scale + n));
        }
      }
    };
    auto sconv = [](uint32_t b) -> float {
      return W4 ? __half2float(__ushort_as_half(static_cast<unsigned short>(b))) : __uint_as_float(b);
    };
    // Codes and scales are loaded two of this group's code fills ahead into named
    // registers: a fill's values are used two fills after their loads were issued, and the
    // rotation moves values loaded one fill earlier, so no instruction waits on a fresh
    // global load.  (Converting the fp16 scale right at its load made every fill wait for
    // it; an indexed array would live in local memory, and storing a just-loaded value
    // there waits for it too.)  A second walk of the units tracks the fill loaded next:
    // s_f counts every fill, so its parity tells the group.
    UnitWalk sw(pair, npairs, ntiles, tile_fills, sk, p.sk_dp_tiles);
    Unit su;
    bool s_more = sw.next(su);
    int s_kb = s_more ? su.f0 : 0;
    long long s_f = 0;
    auto s_advance = [&]() {
      ++s_f;
      if (++s_kb >= su.f1) {
        s_more = sw.next(su);
        if (s_more) s_kb = su.f0;
      }
    };
    auto load_next = [&](FillCodes& q) {
      while (s_more && (s_kb >= nkb || static_cast<int>(s_f & 1) != grp)) s_advance();  // LoRA fills, other group
      if (!s_more) {
        q.s = 0u;
#pragma unroll
        for (int i = 0; i < NW; ++i) q.c[i] = make_uint4(0u, 0u, 0u, 0u);
        return;
      }
      fill_codes(su.t, s_kb, q);
      s_advance();
    };
    FillCodes n1, n2;  // this group's next code fill and the one after
    load_next(n1);
    load_next(n2);
    int stage = 0;
    uint32_t phase = 0;
    UnitWalk w(pair, npairs, ntiles, tile_fills, sk, p.sk_dp_tiles);
    Unit un;
    while (w.next(un)) {
      bool ok = true;
      for (int kb = un.f0; kb < un.f1; ++kb) {
        if ((stage & 1) == grp) {
          const bool code = kb < nkb;
          FillCodes cur;
          if (code) {
            cur = n1;
            n1 = n2;
            load_next(n2);
          }
          // the MMAs of the stage's previous fill completed: its B tile may be rewritten
          // (a LoRA fill waits too, so no group runs a ring ahead of the MMA)
          if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, wc)) { ok = false; break; }
          if (code) {
            const float sc = sconv(cur.s);
            uint8_t* sB = smem + stage * C::STAGE_BYTES + C::A_BYTES;
            // destination: one 128-byte row (64 bf16, 128-byte swizzle: 16-byte unit u at
            // u ^ (row & 7))
            uint8_t* rowp = !B_MN ? sB + row * 128 : sB + h * (C::B_BYTES / 2) + row * 128;
            uint32_t cw[4 * NW];  // the row's codes as 32-bit words, in memory order
#pragma unroll
            for (int i = 0; i < NW; ++i) {
              cw[4 * i] = cur.c[i].x;
              cw[4 * i + 1] = cur.c[i].y;
              cw[4 * i + 2] = cur.c[i].z;
              cw[4 * i + 3] = cur.c[i].w;
            }
            if constexpr (W4) {
              uint32_t L[4], H[4];
              block_levels(cb, sc, L, H);
#pragma unroll
              for (int u = 0; u < 8; ++u)
                *reinterpret_cast<uint4*>(rowp + ((u ^ (row & 7)) << 4)) = expand8(cw[u], L, H);
            } else {
#pragma unroll
              for (int u = 0; u < 8; ++u)
                *reinterpret_cast<uint4*>(rowp + ((u ^ (row & 7)) << 4)) =
                    expand8_w8<WF>(cw[2 * u], cw[2 * u + 1], sc);
            }
            fence_proxy_async_smem();
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&deql[stage]));
        }
        if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
    }
  }

  // the staged output stores of this warp are complete before the CTA exits
  if (EPI == EPI_STORE && C::STAGED_STORE && warp >= 2 && warp < 2 + C::NUM_EPI_WARPS && lane == 0) bulk_wait<0>();

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  __syncwarp();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace lora
