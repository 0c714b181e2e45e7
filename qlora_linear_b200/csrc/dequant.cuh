// dequant.cuh — expansion of quantized weight codes to bf16 inside the GEMM's shared-
// memory staging: the 4-bit blockwise codes (16-level codebook, one fp16 scale per 64
// elements) and the 8-bit int8 / fp8 e4m3 codes with fp32 row scales.  Each element
// becomes bf16_rn(fp32_rn(value(code) * scale)), the same bits the standalone
// dequantization writes.
#pragma once

#include "ptx.cuh"

namespace lora {

// Storage format of the frozen weight (the values of lora_wfmt_t).
enum : int { WF_BF16 = 0, WF_BLOCK4 = 1, WF_INT8 = 2, WF_FP8 = 3 };

// Expands 8 codes (one 32-bit word) of one 64-element scale block to 8 bf16, using the
// block's 16 dequantized levels held as byte planes: low bytes of level e in byte e%4
// of L[e/4], high bytes likewise in H.  Element 2j sits in the low nibble of byte j,
// so the low 16 bits of `w` select elements 0..3.  Each prmt picks four bytes by
// 3-bit selectors; the selector's bit 3 (code >= 8) picks between the two halves.
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

}  // namespace lora
