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
// never formed.  With W4 the frozen weight arrives as packed 4-bit codes ("Rev vs
// unsloth", fused quantized-LoRA paragraph) and each CTA's dequant warps expand them in
// shared memory into the bf16 tile the tensor core reads; no dequantized weight ever
// reaches HBM.
//
// A cluster of two CTAs computes a 256×256 tile.  Each CTA loads its own 128 rows of A
// and its own 128 rows of the B tile (no multicast); the even CTA ("leader") issues
// tcgen05.mma.cta_group::2 (M=256, N=256, K=16), which reads both CTAs' shared memory
// and accumulates into both CTAs' TMEM (each CTA holds its 128 rows × 256 fp32 columns,
// double-buffered).  Per CTA this halves the operand bytes per MMA compared with a
// 128×256 single-CTA tile, and for W4 halves the dequant work per MMA.
//
// Synchronisation.  TMA completions of both CTAs count on the leader's `full` barrier;
// the leader's MMA commits arrive on both CTAs' `empty` / `tfull` barriers (CTA mask
// 0b11); both CTAs' epilogue and dequant warps arrive on the leader's `tempty` / `deq`
// barriers through cluster addresses.  W4 code tiles complete on a CTA-local `cfull`
// barrier so each CTA's dequant warps can wait locally.  Every wait is bounded.
//
// Roles per CTA: warp 0 TMA producer, warp 1 MMA issuer (leader) and TMEM owner,
// warps 2-5 epilogue, warps 6-13 dequant (W4 only).
#pragma once

#include "ptx.cuh"

namespace lora {

struct PairParams {
  int M;               // rows of Aop / out
  int Nout;            // columns of out
  int Kred;            // reduction length (K forward, N backward)
  int r;               // rank of the LoRA fill (<= 128): one extra K fill
  // Grouped projections (forward): output tile columns [seg_end[g-1], seg_end[g]) (in
  // 256-column tiles) belong to segment g, whose E columns start at g * e_seg_stride.
  int nseg;            // 1 for a single projection
  int e_seg_stride;
  int seg_end_tile[8];
  int group_m;         // 256-row tiles per raster group (L2 reuse of the B operand)
  // SwiGLU epilogues (feed-forward block).  Forward: the even CTA of a pair takes gate
  // rows nb*128.., the odd CTA the up rows half_rows further on, and the odd CTA's LoRA
  // F tile starts f_shift columns to the left, so it meets the up half of E.
  int half_rows;
  int f_shift;
  __nv_bfloat16* aux;  // [M, ld_aux]: gate pre-activations, up pre-activations aux_off columns on
  int ld_aux;
  int aux_off;
  // Cross-entropy over an LM head (logits = the GEMM's output columns, vocabulary index
  // v0 + column).
  const int32_t* labels;   // [M]
  int ignore_index;
  int v0;
  float* lse_part;         // EPI_CE_LSE: [num_n][M][2] (max, sum of exp(z - max)) per 256-column tile
  float* label_logit;      // EPI_CE_LSE: [M], written by the tile holding the row's label
  const float* lse;        // EPI_CE_DLOGITS: [M]
  const float* dloss;      // EPI_CE_DLOGITS: [M] upstream gradient of each row's loss
  float* acc32;            // EPI_ACC_F32: [M, Nout] fp32 running sum
  int acc_mode;            // EPI_ACC_F32: bit 0 add the running sum, bit 1 write bf16 to out instead
  __nv_bfloat16* out;  // [M, Nout] row-major
  uint32_t* status;    // device status word, may be null
  uint64_t wait_ns;    // bound of every mbarrier wait
  // quantized weights only
  const __half* absmax;      // 4-bit: fp16 [Nw*Kw/64]
  const float* codebook;     // 4-bit: [16]
  const float* row_scale;    // 8-bit: fp32 [Nw]
  int Nw, Kw;                // logical weight shape [Nw, Kw]
};

// Storage format of the frozen weight (the values of lora_wfmt_t).
enum : int { WF_BF16 = 0, WF_BLOCK4 = 1, WF_INT8 = 2, WF_FP8 = 3 };

template <bool B_MN, int WF>
struct PairCfg {
  static constexpr bool W4 = WF == WF_BLOCK4;
  static constexpr bool W8 = WF == WF_INT8 || WF == WF_FP8;
  static constexpr bool DEQ = W4 || W8;  // the B tile is expanded in shared memory
  static constexpr int BM = 256, BN = 256, BK = 128;  // pair tile, K per pipeline fill
  static constexpr int HM = 128, HN = 128;            // per-CTA halves of A rows / B rows
  static constexpr int STAGES = 3;
  static constexpr int ATOM = 64;                       // 128-byte swizzle atom width (bf16)
  static constexpr int A_BYTES = HM * BK * 2;           // 32 KB (two 64-wide K atoms)
  static constexpr int B_BYTES = HN * BK * 2;           // 32 KB
  static constexpr int C_BYTES = W4 ? HN * BK / 2 : 0;  // 8 KB of codes
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + C_BYTES;
  static constexpr int NUM_EPI_WARPS = 4;
  static constexpr int NUM_DEQ_WARPS = DEQ ? 8 : 0;  // two per SM sub-partition
  static constexpr int NUM_THREADS = 32 * (2 + NUM_EPI_WARPS + NUM_DEQ_WARPS);
  static constexpr int TMEM_COLS = 512;
  static constexpr int NUM_BARS = 4 * STAGES + 5;
  static constexpr int SCALE_RING = 4;  // W4: scale words staged this many code fills ahead (minus one)
  static constexpr int SCALE_BYTES = W4 ? SCALE_RING * 32 * NUM_DEQ_WARPS * 4 : 0;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + SCALE_BYTES + 8 * NUM_BARS + 16;
  static_assert(STAGE_BYTES % 1024 == 0, "stages must keep the 1024-byte swizzle alignment");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// Epilogue of the pair GEMM.
enum : int {
  EPI_STORE = 0,       // out = accumulator (bf16)
  EPI_SWIGLU_FWD = 1,  // accumulator columns [0,128) gate g, [128,256) up u of the same 128
                       // output columns: aux <- g, u; out <- silu(g)·u
  EPI_SWIGLU_BWD = 2,  // accumulator = dH; aux holds g, u and is overwritten in place with
                       // dG = dH·u·silu'(g), dU = dH·silu(g); out is not written
  EPI_CE_LSE = 3,      // accumulator = logits: per row and tile (max, Σ exp(z - max)) and the
                       // label's logit; no logits are written
  EPI_CE_DLOGITS = 4,  // accumulator = logits: out <- dloss·(exp(z - lse) - [label == column])
  EPI_ACC_F32 = 5,     // out/acc32 <- accumulator (+ acc32), see acc_mode
};

template <int EPI>
struct EpiTile {
  static constexpr int COLS = EPI == EPI_SWIGLU_FWD ? 128 : 256;  // output columns per pair tile
};

// First row of this CTA's half of the B tile (and of its LoRA F tile).
template <int EPI>
__device__ __forceinline__ int pair_brow(int nb, uint32_t rank, const PairParams& p) {
  if (EPI == EPI_SWIGLU_FWD) return nb * 128 + static_cast<int>(rank) * p.half_rows;
  return nb * 256 + static_cast<int>(rank) * 128;
}

// silu(g) = g·sigmoid(g); sigmoid from the exponential intrinsic and a rounded reciprocal
// (1/(1+e^-g) is 0, not NaN, when e^-g overflows).
__device__ __forceinline__ float sigmoid_f(float g) { return __frcp_rn(1.0f + __expf(-g)); }

__device__ __forceinline__ void pair_tile_coords(int t, int num_m, int num_n, int group_m, int& mb, int& nb) {
  const int per_group = group_m * num_n;
  const int g = t / per_group;
  const int first_m = g * group_m;
  const int gm = min(group_m, num_m - first_m);
  const int within = t - first_m * num_n;
  mb = first_m + within % gm;
  nb = within / gm;
}

// Expands 8 codes (one 32-bit word) of one 64-element scale block to 8 bf16, using the
// block's 16 dequantized levels held as byte planes: low bytes of level e in byte e%4
// of L[e/4], high bytes likewise in H.  Element 2j sits in the low nibble of byte j,
// so the low 16 bits of `w` select elements 0..3.  Each prmt picks four bytes by
// 3-bit selectors; the selector's bit 3 (code >= 8) picks between the two halves.
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

// The 16 levels of one scale block, bf16_rn(fp32_rn(codebook[c] * scale)), as byte
// planes for expand8().  __fmul_rn keeps the product from being fused with anything.
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

// Eight 8-bit codes (two words, element 4i+j in byte j of word i) to eight bf16
// bf16_rn(fp32_rn(value(code) * scale)).  int8: value = the signed byte, made exact in
// fp32 by placing the biased byte in the mantissa of 2^23; fp8: e4m3 decoded exactly
// through f16 by the hardware conversion.
template <int WF>
__device__ __forceinline__ uint4 expand8_w8(uint32_t w0, uint32_t w1, float sc) {
  float f[8];
  if constexpr (WF == WF_INT8) {
    const uint32_t u0 = w0 ^ 0x80808080u, u1 = w1 ^ 0x80808080u;  // byte + 128, unsigned
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      f[j] = __uint_as_float(prmt(u0, 0x4B000000u, 0x7540u | j)) - 8388736.0f;  // 2^23 + 128
      f[4 + j] = __uint_as_float(prmt(u1, 0x4B000000u, 0x7540u | j)) - 8388736.0f;
    }
  } else {
    const uint32_t hw[4] = {w0 & 0xffffu, w0 >> 16, w1 & 0xffffu, w1 >> 16};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t h2;
      asm("{ .reg .b16 t; cvt.u16.u32 t, %1; cvt.rn.f16x2.e4m3x2 %0, t; }" : "=r"(h2) : "r"(hw[j]));
      const __half2 hv = *reinterpret_cast<const __half2*>(&h2);
      f[2 * j] = __low2float(hv);
      f[2 * j + 1] = __high2float(hv);
    }
  }
  uint4 o;
  o.x = pack_bf16x2(__fmul_rn(f[0], sc), __fmul_rn(f[1], sc));
  o.y = pack_bf16x2(__fmul_rn(f[2], sc), __fmul_rn(f[3], sc));
  o.z = pack_bf16x2(__fmul_rn(f[4], sc), __fmul_rn(f[5], sc));
  o.w = pack_bf16x2(__fmul_rn(f[6], sc), __fmul_rn(f[7], sc));
  return o;
}

template <bool B_MN, int WF, int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairCfg<B_MN, WF>::NUM_THREADS, 1)
    lora_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                          const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmF,
                          const PairParams p) {
  using C = PairCfg<B_MN, WF>;
  constexpr bool W4 = C::W4, W8 = C::W8, DEQ = C::DEQ;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint32_t* scale_ring = reinterpret_cast<uint32_t*>(smem + C::STAGES * C::STAGE_BYTES);  // W4
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES + C::SCALE_BYTES);
  uint64_t* full = bars;                    // leader: TMA bytes of both CTAs landed
  uint64_t* empty = bars + C::STAGES;       // both: the pair MMA finished reading the stage
  uint64_t* cfull = bars + 2 * C::STAGES;   // both (4-/8-bit): this CTA's code tile landed
  uint64_t* deq = bars + 3 * C::STAGES;     // leader (4-/8-bit): both CTAs' dequantized tiles written
  uint64_t* tfull = bars + 4 * C::STAGES;   // both: accumulator ready for the epilogue
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
  const int nkb = (p.Kred + C::BK - 1) / C::BK;
  const int n_ext = p.r > 0 ? 1 : 0;         // one fill holds the whole LoRA block (r <= 128)
  const int ext_atoms = p.r > 64 ? 2 : 1;   // 64-wide rank atoms actually loaded
  const WaitCtl wc{abort_flag, p.status, p.wait_ns};

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
      mbar_init(smem_u32(&cfull[s]), 1);
      mbar_init(smem_u32(&deq[s]), 2 * (C::NUM_DEQ_WARPS > 0 ? C::NUM_DEQ_WARPS : 1));
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&tfull[a]), 1);
      mbar_init(smem_u32(&tempty[a]), 2 * C::NUM_EPI_WARPS);
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
      for (int t = pair; t < ntiles && ok; t += npairs) {
        int mb, nb;
        pair_tile_coords(t, num_m, num_n, p.group_m, mb, nb);
        const int arow = mb * C::BM + static_cast<int>(rank) * C::HM;  // this CTA's rows of A
        const int brow = pair_brow<EPI>(nb, rank, p);  // this CTA's rows of the B tile
        for (int kb = 0; kb < nkb + n_ext; ++kb) {
          if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, wc)) { ok = false; break; }
          const bool ext = kb >= nkb;
          const uint32_t sA = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t sB = sA + C::A_BYTES;
          const uint32_t sC = sB + C::B_BYTES;
          const uint32_t full_l = mapa_shared(smem_u32(&full[stage]), 0);
          if (leader) {
            uint32_t per_cta;
            if (!ext) per_cta = C::A_BYTES + (DEQ ? 0 : C::B_BYTES);
            else per_cta = ext_atoms * (C::A_BYTES / 2) + (B_MN ? C::B_BYTES : ext_atoms * (C::B_BYTES / 2));
            mbar_arrive_expect_tx(smem_u32(&full[stage]), 2 * per_cta);
          }
          // every box is 64 wide × 128 rows; a K-major operand takes one box per
          // 64-wide K atom, an MN-major one (backward weight) one box per 64-wide MN chunk
          if (!ext) {
            tma_load_2d_pair(sA, &tmA, full_l, kb * C::BK, arow);
            tma_load_2d_pair(sA + C::A_BYTES / 2, &tmA, full_l, kb * C::BK + C::ATOM, arow);
            if (W4) {
              mbar_arrive_expect_tx(smem_u32(&cfull[stage]), C::C_BYTES);
              if (!B_MN) tma_load_2d(sC, &tmB, smem_u32(&cfull[stage]), kb * (C::BK / 2), brow);
              else tma_load_2d(sC, &tmB, smem_u32(&cfull[stage]), brow / 2, kb * C::BK);
            } else if (W8) {
              // 8-bit codes, one 32-row × 64-byte box per dequant warp, placed in the upper
              // half of the 4 KB of the B buffer that warp will write, so each warp reads its
              // codes and expands them in place with no other warp involved
              mbar_arrive_expect_tx(smem_u32(&cfull[stage]), C::B_BYTES / 2);
              for (int w = 0; w < 8; ++w) {
                const int hh = w >> 2, rq = (w & 3) * 32;
                const uint32_t dst = sB + hh * (C::B_BYTES / 2) + rq * 128 + 2048;
                if (!B_MN) tma_load_2d(dst, &tmB, smem_u32(&cfull[stage]), kb * C::BK + hh * C::ATOM, brow + rq);
                else tma_load_2d(dst, &tmB, smem_u32(&cfull[stage]), brow + hh * C::ATOM, kb * C::BK + rq);
              }
            } else if (!B_MN) {
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
            if (DEQ) mbar_arrive(smem_u32(&cfull[stage]));  // nothing to dequantize in this fill
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
          if (DEQ) mbar_wait(smem_u32(&cfull[s]), ph, drain_wc);
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
      for (int t = pair; t < ntiles && ok; t += npairs) {
        if (!mbar_wait<true>(smem_u32(&tempty[acc]), acc_phase ^ 1u, wc)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(acc * C::BN);
        for (int kb = 0; kb < nkb + n_ext; ++kb) {
          if (!mbar_wait(smem_u32(&full[stage]), phase, wc)) { ok = false; break; }
          if (DEQ && !mbar_wait<true>(smem_u32(&deq[stage]), phase, wc)) { ok = false; break; }
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
            tc_mma_bf16_pair(d, ad, bd, idesc, (kb > 0 || k > 0) ? 1u : 0u);
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
  } else if (warp < 2 + C::NUM_EPI_WARPS) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int quarter = warp & 3;  // TMEM lane quarter this warp may access
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = pair; t < ntiles; t += npairs) {
      int mb, nb;
      pair_tile_coords(t, num_m, num_n, p.group_m, mb, nb);
      if (!mbar_wait_warp(smem_u32(&tfull[acc]), acc_phase, wc)) break;
      tc_fence_after();
      const int row = mb * C::BM + static_cast<int>(rank) * C::HM + quarter * 32 + lane;
      const uint32_t tbase =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * C::BN);
      if constexpr (EPI == EPI_STORE) {
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
      } else if constexpr (EPI == EPI_SWIGLU_FWD) {
        __nv_bfloat16* hrow = p.out + static_cast<size_t>(row) * p.Nout;
        __nv_bfloat16* grow = p.aux + static_cast<size_t>(row) * p.ld_aux;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          const int col0 = nb * 128 + c * 32;
          if (col0 >= p.Nout) break;  // warp-uniform
          uint32_t g[32], u[32];
          tmem_ld_32x32b_x32(tbase + c * 32, g);
          tmem_ld_32x32b_x32(tbase + 128 + c * 32, u);
          tmem_ld_wait();
          if (row < p.M) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              if (col0 + q * 8 < p.Nout) {
                uint32_t og[4], ou[4], oh[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const float g0 = __uint_as_float(g[q * 8 + 2 * e]), g1 = __uint_as_float(g[q * 8 + 2 * e + 1]);
                  const float u0 = __uint_as_float(u[q * 8 + 2 * e]), u1 = __uint_as_float(u[q * 8 + 2 * e + 1]);
                  og[e] = pack_bf16x2(g0, g1);
                  ou[e] = pack_bf16x2(u0, u1);
                  oh[e] = pack_bf16x2(g0 * sigmoid_f(g0) * u0, g1 * sigmoid_f(g1) * u1);
                }
                *reinterpret_cast<uint4*>(grow + col0 + q * 8) = make_uint4(og[0], og[1], og[2], og[3]);
                *reinterpret_cast<uint4*>(grow + p.aux_off + col0 + q * 8) = make_uint4(ou[0], ou[1], ou[2], ou[3]);
                *reinterpret_cast<uint4*>(hrow + col0 + q * 8) = make_uint4(oh[0], oh[1], oh[2], oh[3]);
              }
            }
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
      } else {
        __nv_bfloat16* grow = p.aux + static_cast<size_t>(row) * p.ld_aux;
#pragma unroll 1
        for (int c = 0; c < C::BN / 32; ++c) {
          const int col0 = nb * C::BN + c * 32;
          if (col0 >= p.Nout) break;  // warp-uniform
          uint32_t v[32];
          tmem_ld_32x32b_x32(tbase + c * 32, v);
          uint4 gq[4], uq[4];
          if (row < p.M) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              if (col0 + q * 8 < p.Nout) {
                gq[q] = *reinterpret_cast<const uint4*>(grow + col0 + q * 8);
                uq[q] = *reinterpret_cast<const uint4*>(grow + p.aux_off + col0 + q * 8);
              }
            }
          }
          tmem_ld_wait();
          if (row < p.M) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              if (col0 + q * 8 < p.Nout) {
                const uint32_t gw[4] = {gq[q].x, gq[q].y, gq[q].z, gq[q].w};
                const uint32_t uw[4] = {uq[q].x, uq[q].y, uq[q].z, uq[q].w};
                uint32_t odg[4], odu[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  float dg[2], du[2];
#pragma unroll
                  for (int h2 = 0; h2 < 2; ++h2) {
                    const float gv = __uint_as_float(h2 ? (gw[e] & 0xffff0000u) : (gw[e] << 16));
                    const float uv = __uint_as_float(h2 ? (uw[e] & 0xffff0000u) : (uw[e] << 16));
                    const float dh = __uint_as_float(v[q * 8 + 2 * e + h2]);
                    const float sg = sigmoid_f(gv);
                    du[h2] = dh * gv * sg;
                    dg[h2] = dh * uv * sg * (1.0f + gv * (1.0f - sg));
                  }
                  odg[e] = pack_bf16x2(dg[0], dg[1]);
                  odu[e] = pack_bf16x2(du[0], du[1]);
                }
                *reinterpret_cast<uint4*>(grow + col0 + q * 8) = make_uint4(odg[0], odg[1], odg[2], odg[3]);
                *reinterpret_cast<uint4*>(grow + p.aux_off + col0 + q * 8) = make_uint4(odu[0], odu[1], odu[2], odu[3]);
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
  } else if constexpr (W4) {
    // ------------------------------------------------------------ dequant (4-bit, both CTAs)
    const int dt = threadIdx.x - 32 * (2 + C::NUM_EPI_WARPS);  // 0..255
    const int row = dt & 127;  // weight row of this CTA's 128-row half (forward) / of the K fill (backward)
    const int h = dt >> 7;     // 64-wide atom: K atom (forward) or output chunk (backward)
    float cb[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) cb[i] = __ldg(p.codebook + i);
    const long long kblocks_w = p.Kw / 64;  // scale blocks per weight row
    const long long nscales = static_cast<long long>(p.Nw) * kblocks_w;
    // Each thread expands one 64-element scale block per code fill.  The fp16 scales
    // are staged in a per-thread shared-memory ring with cp.async, SCALE_RING-1 code
    // fills ahead, so no register ever waits on an outstanding global load.
    const int my_tiles = ntiles > pair ? (ntiles - pair + npairs - 1) / npairs : 0;
    const int code_fills = my_tiles * nkb;  // fills of this CTA that carry codes
    auto stage_scale = [&](int i) {           // issue the copy for code fill i (always commits a group)
      if (i < code_fills) {
        const int t = pair + (i / nkb) * npairs, kb = i % nkb;
        int mb, nb;
        pair_tile_coords(t, num_m, num_n, p.group_m, mb, nb);
        const int brow = pair_brow<EPI>(nb, rank, p);
        const long long n = !B_MN ? brow + row : static_cast<long long>(kb) * C::BK + row;
        const long long kblk = !B_MN ? kb * 2 + h : brow / 64 + h;
        const uint32_t dst = smem_u32(&scale_ring[(i % C::SCALE_RING) * (32 * C::NUM_DEQ_WARPS) + dt]);
        if (n < p.Nw && kblk < kblocks_w) {
          // 4-byte aligned word holding the scale; the half beyond the array end reads as zero
          const long long idx = n * kblocks_w + kblk;
          const long long w0 = idx & ~1LL;
          const uint32_t nbytes = (w0 + 1 < nscales) ? 4u : 2u;
          asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(p.absmax + w0), "r"(nbytes)
                       : "memory");
        } else {
          asm volatile("cp.async.ca.shared.global [%0], [%1], 4, 0;" ::"r"(dst), "l"(p.absmax) : "memory");
        }
      }
      cp_async_commit();
    };
    auto scale_of = [&](int i) -> float {
      int kb = i % nkb, t = pair + (i / nkb) * npairs;
      int mb, nb;
      pair_tile_coords(t, num_m, num_n, p.group_m, mb, nb);
      const int brow = pair_brow<EPI>(nb, rank, p);
      const long long n = !B_MN ? brow + row : static_cast<long long>(kb) * C::BK + row;
      const long long kblk = !B_MN ? kb * 2 + h : brow / 64 + h;
      const uint32_t wv = scale_ring[(i % C::SCALE_RING) * (32 * C::NUM_DEQ_WARPS) + dt];
      const uint16_t hb = ((n * kblocks_w + kblk) & 1) ? static_cast<uint16_t>(wv >> 16) : static_cast<uint16_t>(wv);
      return __half2float(__ushort_as_half(hb));
    };
#pragma unroll 1
    for (int i = 0; i < C::SCALE_RING - 1; ++i) stage_scale(i);
    int stage = 0;
    uint32_t phase = 0;
    int ci = 0;  // index of the next code fill
    for (int t = pair; t < ntiles; t += npairs) {
      bool ok = true;
      for (int kb = 0; kb < nkb + n_ext; ++kb) {
        if (kb < nkb) stage_scale(ci + C::SCALE_RING - 1);
        if (!mbar_wait(smem_u32(&cfull[stage]), phase, wc)) { ok = false; break; }
        if (kb < nkb) {
          cp_async_wait<C::SCALE_RING - 1>();  // this fill's scale word has landed
          const float sc = scale_of(ci);
          ++ci;
          uint8_t* sB = smem + stage * C::STAGE_BYTES + C::A_BYTES;
          const uint8_t* crow = sB + C::B_BYTES + row * 64 + h * 32;  // 32 code bytes = 64 codes
          uint32_t L[4], H[4];
          block_levels(cb, sc, L, H);
          const uint4 c0 = *reinterpret_cast<const uint4*>(crow);
          const uint4 c1 = *reinterpret_cast<const uint4*>(crow + 16);
          const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
          uint8_t* rowp = sB + h * (C::B_BYTES / 2) + row * 128;
#pragma unroll
          for (int u = 0; u < 8; ++u)
            *reinterpret_cast<uint4*>(rowp + ((u ^ (row & 7)) << 4)) = expand8(cw[u], L, H);
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&deq[stage]), 0));
        if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
    }
    cp_async_wait<0>();  // no copy may still target shared memory at exit
  } else if constexpr (W8) {
    // ------------------------------------------------------------ dequant (8-bit, both CTAs)
    const int dt = threadIdx.x - 32 * (2 + C::NUM_EPI_WARPS);  // 0..255
    const int row = dt & 127;  // weight row of this CTA's half (forward) / of the K fill (backward)
    const int h = dt >> 7;     // 64-wide atom: K atom (forward) or output chunk (backward)
    // fp32 scale of the weight row this thread expands in code fill (t, kb)
    auto scale_at = [&](int t, int kb) -> float {
      int mb, nb;
      pair_tile_coords(t, num_m, num_n, p.group_m, mb, nb);
      const long long n = !B_MN ? static_cast<long long>(pair_brow<EPI>(nb, rank, p)) + row
                                : static_cast<long long>(kb) * C::BK + row;
      return n < p.Nw ? __ldg(p.row_scale + n) : 0.0f;
    };
    float sc_next = (pair < ntiles && nkb > 0) ? scale_at(pair, 0) : 0.0f;
    int stage = 0;
    uint32_t phase = 0;
    for (int t = pair; t < ntiles; t += npairs) {
      bool ok = true;
      for (int kb = 0; kb < nkb + n_ext; ++kb) {
        float sc = 0.0f;
        if (kb < nkb) {
          sc = sc_next;  // the next code fill's scale is loaded one fill ahead
          const int tn = kb + 1 < nkb ? t : t + npairs;
          if (tn < ntiles) sc_next = scale_at(tn, kb + 1 < nkb ? kb + 1 : 0);
        }
        if (!mbar_wait(smem_u32(&cfull[stage]), phase, wc)) { ok = false; break; }
        if (kb < nkb) {
          uint8_t* rowp = smem + stage * C::STAGE_BYTES + C::A_BYTES + h * (C::B_BYTES / 2) + row * 128;
          const uint8_t* crow = rowp - (row & 31) * 128 + 2048 + (row & 31) * 64;  // this warp's code box
          uint32_t cw[16];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const uint4 c = *reinterpret_cast<const uint4*>(crow + 16 * u);
            cw[4 * u] = c.x;
            cw[4 * u + 1] = c.y;
            cw[4 * u + 2] = c.z;
            cw[4 * u + 3] = c.w;
          }
          __syncwarp();  // the warp's codes are all in registers before its rows are overwritten
#pragma unroll
          for (int u = 0; u < 8; ++u)
            *reinterpret_cast<uint4*>(rowp + ((u ^ (row & 7)) << 4)) = expand8_w8<WF>(cw[2 * u], cw[2 * u + 1], sc);
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&deq[stage]), 0));
        if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
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
