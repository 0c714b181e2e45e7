// gemm_common.cuh — what the two tcgen05 GEMM kernels share: the launch parameters,
// the tile order, the epilogue modes and their per-chunk arithmetic.
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
  // Stream-K schedule (EPI_STORE only, see UnitWalk): sk_on != 0 runs the first
  // sk_dp_tiles tiles whole and cuts the fill sequence of the rest into one range per CTA
  // pair; pieces of tiles go to the fp32 slots kpart [2 · pairs][tile rows][256].
  int sk_on;
  int sk_dp_tiles;
  float* kpart;
  uint32_t* status;    // device status word, may be null
  uint64_t wait_ns;    // bound of every mbarrier wait
  // quantized weights only
  const __half* absmax;      // 4-bit: fp16 [Nw*Kw/64]
  const float* codebook;     // 4-bit: [16]
  const float* row_scale;    // 8-bit: fp32 [Nw]
  const uint8_t* codes;      // [Nw][Kw/2] (4-bit, two codes a byte) or [Nw][Kw] (8-bit)
  int Nw, Kw;                // logical weight shape [Nw, Kw]
};

// Epilogue of the GEMMs.
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

// Work units of a launch, walked in the same order by every role of a CTA pair.
// A unit is fills [f0, f1) of output tile t, out of the tile's L = nkb + n_ext fills (the
// code fills of the reduction, then the LoRA fills), and either covers the tile whole
// (slot < 0: the epilogue writes the output) or is a piece whose fp32 accumulator goes to
// slot `slot` of kpart.
//   Data-parallel (sk off): pair p takes tiles p, p + P, p + 2P, ... whole.
//   Stream-K (sk on): pair p takes tiles p, p + P, ... below dp_tiles (a multiple of P)
//   whole, then range [p·F/P, (p+1)·F/P) of the F = (ntiles − dp_tiles)·L fills of the
//   remaining tiles laid end to end.  The pair's first piece goes to slot 2p, its last to
//   slot 2p + 1 (a range inside one tile is a single piece in slot 2p); every range holds
//   at least one fill, so the pieces of a tile are those of consecutive pairs.
struct Unit {
  int t, f0, f1, slot;
};
struct UnitWalk {
  int p, P, ntiles, L, dp_left, k;
  long long g, g0, g1;
  bool sk;
  __device__ __forceinline__ UnitWalk(int p_, int P_, int ntiles_, int L_, bool sk_, int dp_tiles)
      : p(p_), P(P_), ntiles(ntiles_), L(L_), dp_left(sk_ ? dp_tiles / P_ : 0), k(0), g(0), g0(0), g1(0), sk(sk_) {
    if (sk) {
      const long long F = static_cast<long long>(ntiles - dp_tiles) * L;
      g0 = static_cast<long long>(p) * F / P;
      g1 = static_cast<long long>(p + 1) * F / P;
      g = g0;
    }
  }
  __device__ __forceinline__ bool next(Unit& u) {
    if (!sk || k < dp_left) {
      const int t = p + k * P;
      if (t >= ntiles) return false;
      ++k;
      u = Unit{t, 0, L, -1};
      return true;
    }
    if (g >= g1) return false;
    const long long tr = g / L;
    const int f0 = static_cast<int>(g - tr * L);
    const int f1 = static_cast<int>(min(static_cast<long long>(L), f0 + (g1 - g)));
    const int slot = (f0 == 0 && f1 == L) ? -1 : (g == g0 ? 2 * p : 2 * p + 1);
    u = Unit{dp_left * P + static_cast<int>(tr), f0, f1, slot};
    g += f1 - f0;
    return true;
  }
};

// ---------------------------------------------------------------- epilogue pieces
// 32 accumulator columns of tile-local row lrow, columns [lc0, lc0 + 32), to a stream-K
// slot (tile-shaped: TILE_ROWS × 256 fp32).
template <int TILE_ROWS>
__device__ __forceinline__ void epi_slot_chunk(const PairParams& p, const uint32_t (&v)[32], int slot, int lrow, int lc0) {
  float* d = p.kpart + (static_cast<size_t>(slot) * TILE_ROWS + lrow) * 256 + lc0;
#pragma unroll
  for (int q = 0; q < 8; ++q)
    reinterpret_cast<float4*>(d)[q] = make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                                  __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
}

// 32 accumulator columns of one row to bf16 out[row, col0 ..].
__device__ __forceinline__ void epi_store_chunk(const PairParams& p, const uint32_t (&v)[32], int row, int col0) {
  __nv_bfloat16* orow = p.out + static_cast<size_t>(row) * p.Nout;
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

// SwiGLU forward: gate g and up u of 32 output columns -> aux (g, u) and out silu(g)·u.
__device__ __forceinline__ void epi_swiglu_fwd_chunk(const PairParams& p, const uint32_t (&g)[32],
                                                     const uint32_t (&u)[32], int row, int col0) {
  __nv_bfloat16* hrow = p.out + static_cast<size_t>(row) * p.Nout;
  __nv_bfloat16* grow = p.aux + static_cast<size_t>(row) * p.ld_aux;
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

// SwiGLU backward: the saved g and u of 32 columns (loaded one chunk ahead of use) ...
struct GU32 {
  uint4 g[4], u[4];
};
__device__ __forceinline__ void epi_swiglu_bwd_load(const PairParams& p, int row, int col0, GU32& x) {
  const __nv_bfloat16* grow = p.aux + static_cast<size_t>(row) * p.ld_aux;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    if (col0 + q * 8 < p.Nout) {
      x.g[q] = *reinterpret_cast<const uint4*>(grow + col0 + q * 8);
      x.u[q] = *reinterpret_cast<const uint4*>(grow + p.aux_off + col0 + q * 8);
    }
  }
}

// ... and dH of the same columns: aux (g, u) overwritten with dG = dH·u·silu'(g), dU = dH·silu(g).
__device__ __forceinline__ void epi_swiglu_bwd_chunk(const PairParams& p, const uint32_t (&v)[32], int row, int col0,
                                                     const GU32& x) {
  __nv_bfloat16* grow = p.aux + static_cast<size_t>(row) * p.ld_aux;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    if (col0 + q * 8 < p.Nout) {
      const uint32_t gw[4] = {x.g[q].x, x.g[q].y, x.g[q].z, x.g[q].w};
      const uint32_t uw[4] = {x.u[q].x, x.u[q].y, x.u[q].z, x.u[q].w};
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

// The SwiGLU-backward epilogue of one row over 32-column chunks [c_begin, c_end) of a
// 256-column accumulator at tbase: the saved g, u of chunk c + 1 are loaded while chunk c
// is converted, two chunks per step so both register sets stay named (the range holds an
// even number of chunks).
__device__ __forceinline__ void epi_swiglu_bwd_row(const PairParams& p, uint32_t tbase, int row, int colbase,
                                                   int c_begin = 0, int c_end = 8) {
  const bool in = row < p.M;
  GU32 x0, x1;
  if (in && colbase + c_begin * 32 < p.Nout) epi_swiglu_bwd_load(p, row, colbase + c_begin * 32, x0);
#pragma unroll 1
  for (int c = c_begin; c < c_end; c += 2) {
    const int col0 = colbase + c * 32, col1 = col0 + 32;
    if (col0 >= p.Nout) break;  // warp-uniform
    if (in && col1 < p.Nout) epi_swiglu_bwd_load(p, row, col1, x1);
    uint32_t v[32];
    tmem_ld_32x32b_x32(tbase + c * 32, v);
    tmem_ld_wait();
    if (in) epi_swiglu_bwd_chunk(p, v, row, col0, x0);
    if (col1 >= p.Nout) break;
    if (in && col1 + 32 < p.Nout && c + 2 < c_end) epi_swiglu_bwd_load(p, row, col1 + 32, x0);
    tmem_ld_32x32b_x32(tbase + (c + 1) * 32, v);
    tmem_ld_wait();
    if (in) epi_swiglu_bwd_chunk(p, v, row, col1, x1);
  }
}

}  // namespace lora
