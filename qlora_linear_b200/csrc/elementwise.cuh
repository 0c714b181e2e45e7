// elementwise.cuh — standalone dequantization (4-bit and 8-bit) and the adapter merge.
//
// Both are HBM-bound and sit outside the forward/backward: the forward and backward
// dequantize tiles in shared memory and never write a dequantized weight to HBM.
#pragma once

#include "ptx.cuh"

namespace lora {

// One element: bf16_rn(fp32_rn(codebook[code] * scale)); the product uses __fmul_rn so
// it can never be contracted into an FMA.
__device__ __forceinline__ float dq_level(const float* lut, uint32_t code, float scale) {
  return __fmul_rn(lut[code], scale);
}

// W_out[N*K] (bf16) from packed codes [N, K/2] and fp16 scales [N*K/64].  Each thread
// expands 16 elements (8 code bytes -> 32 output bytes) per grid-stride step.
__global__ void dequant4_kernel(const uint8_t* __restrict__ codes, const __half* __restrict__ absmax,
                                const float* __restrict__ codebook, __nv_bfloat16* __restrict__ out,
                                size_t total /* N*K */) {
  __shared__ float lut[16];
  if (threadIdx.x < 16) lut[threadIdx.x] = codebook[threadIdx.x];
  __syncthreads();
  const size_t groups = total / 16;
  for (size_t g = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; g < groups;
       g += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const uint2 c = *reinterpret_cast<const uint2*>(codes + g * 8);
    const float sc = __half2float(absmax[(g * 16) / 64]);
    uint32_t w[2] = {c.x, c.y};
    uint32_t o[8];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const uint32_t byte = (w[h] >> (8 * b)) & 0xFFu;
        o[h * 4 + b] = pack_bf16x2(dq_level(lut, byte & 0xFu, sc), dq_level(lut, byte >> 4, sc));
      }
    uint4* dst = reinterpret_cast<uint4*>(out + g * 16);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

// Value of one 8-bit code: the signed byte (int8) or the e4m3 number (fp8), exact in fp32.
template <int WF8>
__device__ __forceinline__ float w8_value(uint32_t byte) {
  if constexpr (WF8 == 2) {
    return static_cast<float>(static_cast<int8_t>(static_cast<uint8_t>(byte)));
  } else {
    uint32_t h2;
    asm("{ .reg .b16 t; cvt.u16.u32 t, %1; cvt.rn.f16x2.e4m3x2 %0, t; }" : "=r"(h2) : "r"(byte & 0xFFu));
    return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
  }
}

// W_out[N*K] (bf16) from 8-bit codes [N, K] and fp32 row scales [N]: each thread expands
// 16 elements (16 code bytes -> 32 output bytes) per grid-stride step (K % 16 == 0).
template <int WF8>
__global__ void dequant8_kernel(const uint8_t* __restrict__ codes, const float* __restrict__ scale,
                                __nv_bfloat16* __restrict__ out, size_t total, long long K) {
  const size_t groups = total / 16;
  for (size_t g = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; g < groups;
       g += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const uint4 c = *reinterpret_cast<const uint4*>(codes + g * 16);
    const float sc = scale[static_cast<long long>(g * 16) / K];
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      o[2 * i] = pack_bf16x2(__fmul_rn(w8_value<WF8>(w[i]), sc), __fmul_rn(w8_value<WF8>(w[i] >> 8), sc));
      o[2 * i + 1] = pack_bf16x2(__fmul_rn(w8_value<WF8>(w[i] >> 16), sc), __fmul_rn(w8_value<WF8>(w[i] >> 24), sc));
    }
    uint4* dst = reinterpret_cast<uint4*>(out + g * 16);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

// W_out = W + s·B·A over a tile of 32 rows × 256 columns per CTA (256 threads, each
// 8 rows × 4 columns), fp32 accumulation.  W is bf16 [N,K] (fmt 0, w16), the 4-bit
// format (fmt 1, codes/absmax/codebook) or 8-bit codes with row scales (fmt 2 int8, 3
// fp8 e4m3; codes/row_scale).  W_out may alias w16: every element is read and then
// written by the same thread.
constexpr int MG_TN = 32, MG_TK = 256, MG_THREADS = 256;

__global__ void __launch_bounds__(MG_THREADS)
    merge_kernel(int fmt, const __nv_bfloat16* w16, const uint8_t* __restrict__ codes,
                 const __half* __restrict__ absmax, const float* __restrict__ codebook,
                 const float* __restrict__ row_scale, const __nv_bfloat16* __restrict__ A,
                 const __nv_bfloat16* __restrict__ B, int N, int K, int r, float s, __nv_bfloat16* out) {
  extern __shared__ __align__(16) float mg_smem[];
  float* sB = mg_smem;                 // [MG_TN][r]
  float* sA = mg_smem + MG_TN * r;     // [r][MG_TK]
  __shared__ float lut[16];
  const int n0 = blockIdx.y * MG_TN, k0 = blockIdx.x * MG_TK;
  if (fmt == 1 && threadIdx.x < 16) lut[threadIdx.x] = codebook[threadIdx.x];
  for (int i = threadIdx.x; i < MG_TN * r; i += MG_THREADS) {
    const int n = n0 + i / r, j = i % r;
    sB[i] = n < N ? __bfloat162float(B[static_cast<size_t>(n) * r + j]) : 0.f;
  }
  for (int i = threadIdx.x; i < r * MG_TK; i += MG_THREADS) {
    const int j = i / MG_TK, k = k0 + i % MG_TK;
    sA[i] = k < K ? __bfloat162float(A[static_cast<size_t>(j) * K + k]) : 0.f;
  }
  __syncthreads();
  const int tk = threadIdx.x % 64, tn = threadIdx.x / 64;  // 64 × 4 threads
  float acc[8][4];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
  for (int j = 0; j < r; ++j) {
    float av[4], bv[8];
#pragma unroll
    for (int b = 0; b < 4; ++b) av[b] = sA[j * MG_TK + tk + 64 * b];
#pragma unroll
    for (int a = 0; a < 8; ++a) bv[a] = sB[(tn + 4 * a) * r + j];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(bv[a], av[b], acc[a][b]);
  }
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    const int n = n0 + tn + 4 * a;
    if (n >= N) continue;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int k = k0 + tk + 64 * b;
      if (k >= K) continue;
      const size_t idx = static_cast<size_t>(n) * K + k;
      float w;
      if (fmt == 0) {
        w = __bfloat162float(w16[idx]);
      } else if (fmt == 1) {
        const uint8_t byte = codes[idx >> 1];
        const uint32_t code = (idx & 1) ? (byte >> 4) : (byte & 0xFu);
        w = __bfloat162float(__float2bfloat16_rn(dq_level(lut, code, __half2float(absmax[idx / 64]))));
      } else {
        const float v = fmt == 2 ? w8_value<2>(codes[idx]) : w8_value<3>(codes[idx]);
        w = __bfloat162float(__float2bfloat16_rn(__fmul_rn(v, row_scale[n])));
      }
      out[idx] = __float2bfloat16_rn(w + s * acc[a][b]);
    }
  }
}

// Cross-entropy: one thread per row combines the per-tile (max, Σ exp(z - max)) partials
// in tile order: lse = m + log Σ_t s_t·exp(m_t - m) with m = max_t m_t, and
// loss = lse - z_label (0 for an ignored row).
__global__ void ce_finalize_kernel(const float2* __restrict__ part, int ntiles, int M,
                                   const float* __restrict__ label_logit, const int32_t* __restrict__ labels,
                                   int ignore_index, float* __restrict__ loss, float* __restrict__ lse) {
  griddep_enter();  // the previous kernel in the stream completed (see ptx.cuh)
  const int row = blockIdx.x * blockDim.x + threadIdx.x;
  if (row >= M) return;
  float m = -INFINITY;
  for (int t = 0; t < ntiles; ++t) m = fmaxf(m, part[static_cast<size_t>(t) * M + row].x);
  float sum = 0.0f;
  for (int t = 0; t < ntiles; ++t) {
    const float2 q = part[static_cast<size_t>(t) * M + row];
    if (q.x != -INFINITY) sum += q.y * expf(q.x - m);
  }
  const float l = m + logf(sum);
  lse[row] = l;
  loss[row] = labels[row] == ignore_index ? 0.0f : l - label_logit[row];
}

// Test hook: waits on an mbarrier that nothing arrives on, with the library's bounded
// wait, so the host can check that an expired wait ends the kernel and sets the status.
__global__ void bounded_wait_probe_kernel(uint32_t* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t flags[2];
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    flags[0] = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitCtl w{reinterpret_cast<volatile uint32_t*>(&flags[0]), status, limit_ns};
    mbar_wait(smem_u32(&bar), 0, w);
  }
}

}  // namespace lora
