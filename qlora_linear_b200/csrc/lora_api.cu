// lora_api.cu — host side of liblora_linear.so: argument validation, workspace layout,
// TMA descriptors, kernel launches and the exported C ABI (include/lora_linear.h).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdlib>
#include <cstring>
#include <atomic>
#include <mutex>
#include <utility>
#include <vector>

#include "lora_linear.h"
#include "lora_linear_profiling.h"
#include "lora_linear_testing.h"
#include "dualproj.cuh"
#include "elementwise.cuh"
#include "gemm_pair.cuh"
#include "gemm_q.cuh"
#include "skinny.cuh"
#include "streamk.cuh"
#include "tcproj.cuh"

namespace lora {
namespace {

constexpr int kTargetCtas = 296;          // skinny passes: about two waves of 148 SMs
constexpr uint64_t kDefaultWaitNs = 2000000000ull;  // 2 s bound for every device wait
constexpr size_t kStatusBytes = 256;      // workspace head: device status word

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
inline int cdiv(long long a, long long b) { return static_cast<int>((a + b - 1) / b); }

uint64_t wait_limit_ns() {
  static uint64_t v = [] {
    const char* e = std::getenv("LORA_WAIT_LIMIT_NS");
    if (e && *e) {
      const unsigned long long x = std::strtoull(e, nullptr, 10);
      if (x > 0) return static_cast<uint64_t>(x);
    }
    return kDefaultWaitNs;
  }();
  return v;
}

// 256-row output tiles per raster group of the GEMMs; LORA_GROUP_M overrides (1..64).
// The tiles of a group walk the output column by column, re-reading the group's A panels
// (256 × Kred bf16 each) from L2 for every column.  16 keeps a reduction-over-4096
// launch at ~1.2 GB of DRAM traffic (0.77 GB read; ~1.1 GB read with 8).  A reduction
// over 14336 reads 2.5-3.4 GB with either 8 or 16: the group's panels and the 117 MB
// weight exceed the 126 MB L2 whatever the group, and the pairs drift apart in k over the
// 14 waves.  16 was ~1.4% faster than 8 in 100-step power-capped runs of the c2 step.
int group_m_default() {
  static int v = [] {
    const char* e = std::getenv("LORA_GROUP_M");
    if (e && *e) {
      const long x = std::strtol(e, nullptr, 10);
      if (x >= 1 && x <= 64) return static_cast<int>(x);
    }
    return 16;
  }();
  return v;
}

// ---------------------------------------------------------------- measurement hooks
std::atomic<long long> g_launches{0};
std::atomic<bool> g_timing_on{false};
std::mutex g_timing_mu;
std::vector<std::pair<cudaEvent_t, cudaEvent_t>> g_timing[LORA_KERNEL_COUNT];

inline void count_launch(int n = 1) { g_launches.fetch_add(n, std::memory_order_relaxed); }

struct TimedRegion {
  cudaEvent_t a = nullptr, b = nullptr;
  cudaStream_t st;
  int kind;
  TimedRegion(int k, cudaStream_t s) : st(s), kind(k) {
    if (!g_timing_on.load(std::memory_order_relaxed)) return;
    if (cudaEventCreate(&a) != cudaSuccess || cudaEventCreate(&b) != cudaSuccess) {
      a = b = nullptr;
      return;
    }
    cudaEventRecord(a, st);
  }
  ~TimedRegion() {
    if (!a) return;
    cudaEventRecord(b, st);
    std::lock_guard<std::mutex> lk(g_timing_mu);
    g_timing[kind].emplace_back(a, b);
  }
};

// ---------------------------------------------------------------- kernel launch
// The layer's kernels are launched with programmatic stream serialization: a kernel may
// start launching while the previous kernel in the stream finishes (its CTA set-up
// overlaps that kernel's tail); each waits (griddepcontrol.wait) for the previous grid to
// complete before its first global-memory access, so the stream order of every read and
// write is kept.  LORA_PDL=0 launches them plainly.
bool pdl_enabled() {
  static bool v = [] {
    const char* e = std::getenv("LORA_PDL");
    return !(e && e[0] == '0');
  }();
  return v;
}
template <typename... Params, typename... Args>
void launch_k(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // a launch error stays pending for cudaGetLastError (last_launch) like one of <<<>>>
  (void)cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------- split heuristics
// Pure functions of the sizes, so the workspace size and the summation order are
// fixed by the problem alone.
struct Split {
  int splits;
  int tiles_per_split;
};
Split make_split(int blocks, int tiles) {
  if (tiles <= 0) return Split{1, 1};
  int want = cdiv(kTargetCtas, blocks > 0 ? blocks : 1);
  int cap = tiles / 2 > 1 ? tiles / 2 : 1;
  int s = want < cap ? want : cap;
  if (s < 1) s = 1;
  const int per = cdiv(tiles, s);
  return Split{cdiv(tiles, per), per};
}
Split rowproj_split(long long M, long long Kred) {
  return make_split(cdiv(M, SK_BM), cdiv(Kred, SK_BK));
}
Split colproj_split(long long M, long long Kout) {
  return make_split(cdiv(Kout, SK_BM), cdiv(M, SK_BK));
}

// Blocking of the one-pass dY·B / dYᵀ·XA kernel: a × b blocks of row_tiles × col_tiles
// tiles, one CTA per SM (its shared memory), at most one wave.  The cost model counts
// the slowest block's bytes at the rate of an even share of HBM (below ~136 CTAs a CTA
// cannot pull more than that share: measured streaming rates fall off below that) plus
// the partials written and read back; the two separate passes stream dY twice at ~0.8 of
// this kernel's rate.
constexpr int kDualCtas = 148;
struct DualSplit {
  bool use = false;
  int a = 0, b = 0, row_tiles = 0, col_tiles = 0;
};
DualSplit dual_split(long long M, long long C, int r, int mode = DP_BOTH) {
  DualSplit best;
  if (r > DP_RPAD || M <= 0 || C <= 0) return best;
  const int ntr = cdiv(M, DP_TR), ntc = cdiv(C, DP_TC);
  const double tile = double(DP_TR) * DP_TC * 2;
  // against the cp.async passes: two of them for both products, one for a single product
  double best_cost = (mode == DP_BOTH ? 2.4 : 1.2) * ntr * double(ntc) * tile;
  const double wT = mode == DP_COLS ? 0.0 : 1.0, wD = mode == DP_ROWS ? 0.0 : 1.0;
  for (int rt = 1; rt <= DP_MAX_ROW_TILES && rt <= ntr; ++rt) {
    const int a = cdiv(ntr, rt);
    if (a > kDualCtas) continue;
    for (int ct = 1; ct <= ntc; ++ct) {
      const int b = cdiv(ntc, ct);
      if (static_cast<long long>(a) * b > kDualCtas) continue;
      const int n = a * b;
      const double cost = double(rt) * ct * tile * (n > 136 ? n : 136) + 2.0 * (wD * a * C + wT * b * M) * r * 4;
      if (cost < best_cost) {
        best_cost = cost;
        best = DualSplit{true, a, b, rt, ct};
      }
    }
  }
  return best;
}
size_t dual_part_t_bytes(const DualSplit& d, long long M, int r) {
  return align256(static_cast<size_t>(d.b) * M * r * 4);
}
size_t dual_part_d_bytes(const DualSplit& d, long long C, int r) {
  return align256(static_cast<size_t>(d.a) * C * r * 4);
}
size_t dual_part_bytes(const DualSplit& d, long long M, long long C, int r) {
  return d.use ? dual_part_t_bytes(d, M, r) + align256(static_cast<size_t>(d.a) * C * r * 4) : 0;
}

// Schedule of a GEMM launch.  Whole tiles round-robin over the CTA pairs leave pairs
// idle in the last wave when the tile count is not a multiple of the pairs (an output of
// 1.5 waves runs two full ones).  Stream-K evens that out: every pair first runs the same
// number of whole tiles, then an equal share of the fills of the remaining tiles, pieces
// of tiles going to fp32 slots that a second kernel adds in pair order (deterministic).
// The whole tiles are either all full waves (only the partial last wave is cut) or all
// full waves but one (the last full wave is cut too, for longer ranges); of the two the
// model takes the cheaper.  The choice is a pure function of the sizes, the rank and the
// weight's format (its tile shape), made against a fixed 74 pairs, so the workspace size
// follows from the sizes alone.  Cost model: fills per pair at the kernel's per-pair
// rate (plus three for the extra epilogue of a piece), slots (about one per cut tile and
// one per pair) written and read back at 5 TB/s, and the fixup launch; stream-K must
// save 3%, and every pair's range holds at least four fills.
constexpr int kGemmPairs = 74;
struct GemmSched {
  bool sk = false;
  int dp_tiles = 0;
  int tile_rows = 256;
  int tile_fills = 0;
};
GemmSched gemm_sched(long long M, long long Nout, long long Kred, int r, bool quantized) {
  GemmSched g;
  g.tile_rows = quantized ? 512 : 256;
  if (M <= 0 || Nout <= 0 || Kred <= 0) return g;
  const int bk = quantized ? 64 : 128;
  const long long tiles = static_cast<long long>(cdiv(M, g.tile_rows)) * cdiv(Nout, 256);
  const long long L = cdiv(Kred, bk) + (r > 0 ? (quantized ? cdiv(r, 64) : 1) : 0);
  g.tile_fills = static_cast<int>(L);
  const int P = kGemmPairs;
  const long long full = tiles / P;
  const double fill_s = 2.0 * g.tile_rows * 256 * bk / ((quantized ? 1.2e15 : 1.5e15) / P);
  const double slot_bytes = double(g.tile_rows) * 256 * 4;
  const double t_dp = double((tiles + P - 1) / P) * L * fill_s;
  double best = 0.97 * t_dp;
  for (long long waves = full > 1 ? full - 1 : 0; waves <= full; ++waves) {
    const long long dp = waves * P;
    const long long rest = tiles - dp;
    if (rest <= 0 || rest * L < 4LL * P) continue;
    const double t_sk = (double(waves) * L + double((rest * L + P - 1) / P) + 3.0) * fill_s +
                        2.0 * double(rest + P) * slot_bytes / 5.0e12 + 4.0e-6;
    if (t_sk < best) {
      best = t_sk;
      g.sk = true;
      g.dp_tiles = static_cast<int>(dp);
    }
  }
  return g;
}
// Split of a tensor-core rank-r pass (ranks above 16): output tiles of 128 rows and the
// number of splits of the reduction that minimises the estimated time in 64-deep fills:
// (waves of two CTAs per SM) × (fills per split + 3 for a CTA's ramp-up and epilogue)
// plus the fp32 partials written and read back (2·splits·rows·r·4 bytes) at the bytes one
// fill of every resident CTA streams (296 × 16 KB).  A second, mostly empty wave costs as
// much as a full one.  Splits hold at least four fills, none is empty.  A pure function of
// the sizes (made for 148 SMs).
struct TcSplit {
  int tiles = 0, splits = 1, fps = 1;
};
TcSplit tc_split(long long rows, long long red, int r) {
  TcSplit t;
  t.tiles = cdiv(rows, TP_BM);
  const int nkb = cdiv(red, TP_BK);
  if (t.tiles <= 0 || nkb <= 0) return t;
  constexpr int kResident = 2 * 148;
  const double fill_bytes = kResident * static_cast<double>(TP_P_BYTES);
  const int cap = nkb / 4 > 1 ? nkb / 4 : 1;
  double best = -1.0;
  for (int s = 1; s <= cap && s <= 256; ++s) {
    const int fps = cdiv(nkb, s);
    const int splits = cdiv(nkb, fps);
    const double waves = cdiv(static_cast<long long>(t.tiles) * splits, kResident);
    const double cost = waves * (fps + 3) + 2.0 * splits * static_cast<double>(rows) * r * 4 / fill_bytes;
    if (best < 0 || cost < best) {
      best = cost;
      t.fps = fps;
      t.splits = splits;
    }
  }
  return t;
}
inline bool tc_rank(int r) { return r > 16; }
size_t tc_part_bytes(long long rows, long long red, int r) {
  return align256(static_cast<size_t>(tc_split(rows, red, r).splits) * rows * r * 4);
}

size_t gemm_sched_bytes(long long M, long long Nout, long long Kred, int r, bool quantized) {
  const GemmSched g = gemm_sched(M, Nout, Kred, r, quantized);
  return g.sk ? static_cast<size_t>(2) * kGemmPairs * g.tile_rows * 256 * 4 : 0;
}

struct WsLayout {
  size_t skinny_off, part_off, total;
};
WsLayout ws_layout(long long M, long long N, long long K, int r1, int nseg, bool quantized) {
  WsLayout w;
  const int r = nseg * r1;
  w.skinny_off = kStatusBytes;
  const size_t skinny = align256(static_cast<size_t>(M) * r * 2);
  w.part_off = w.skinny_off + skinny;
  size_t part = 0;
  auto upd = [&](size_t b) { part = b > part ? b : part; };
  upd(static_cast<size_t>(rowproj_split(M, K).splits) * M * r * 4);  // XA
  upd(static_cast<size_t>(rowproj_split(M, N).splits) * M * r * 4);  // dY·B
  upd(static_cast<size_t>(colproj_split(M, N).splits) * N * r * 4);  // dB
  upd(static_cast<size_t>(colproj_split(M, K).splits) * K * r * 4);  // dA
  upd(dual_part_bytes(dual_split(M, N, r1), M, N, r1));              // dY·B and dYᵀ·XA in one pass
  const DualSplit xr = dual_split(M, K, r, DP_ROWS), xc = dual_split(M, K, r, DP_COLS);
  if (xr.use) upd(dual_part_t_bytes(xr, M, r));                      // X·Aᵀ on the TMA stream
  if (xc.use) upd(dual_part_d_bytes(xc, K, r));                      // Xᵀ·(s·dY·B) on the TMA stream
  upd(gemm_sched_bytes(M, N, K, r1, quantized));                    // Y GEMM stream-K slots
  upd(gemm_sched_bytes(M, K, N, r, quantized));                      // dX GEMM stream-K slots
  if (tc_rank(r)) {
    upd(tc_part_bytes(M, K, r));   // X·Aᵀ on the tensor cores
    upd(tc_part_bytes(K, M, r));   // Xᵀ·(s·dY·B) for dA
  }
  if (tc_rank(r1)) {
    upd(tc_part_bytes(M, N, r1));  // dY·B (any segment has at most N rows)
    upd(tc_part_bytes(N, M, r1));  // dYᵀ·XA for dB
  }
  w.total = w.part_off + align256(part);
  return w;
}

// ---------------------------------------------------------------- device info
// The current CUDA context (driver API, looked up through the runtime).  Per-device
// state cached by this library (kernel attributes, the device address of the fixed
// scratch of lora_linear_fwd_noalloc) belongs to one context: after cudaDeviceReset
// the primary context is created anew and that state is set up again.
PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;

// The context current on this thread, or nullptr when none is (yet).
CUcontext current_ctx() {
  static std::once_flag once;
  std::call_once(once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &fn, 4000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess && fn)
      g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
  });
  CUcontext c = nullptr;
  if (!g_ctx_current || g_ctx_current(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

struct DevInfo {
  int sms = 0;
  bool attrs_set = false;
  CUcontext ctx = nullptr;  // context the attributes were set in
};
std::mutex g_mu;
DevInfo g_dev[64];

lora_status_t dev_info(DevInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return LORA_ERR_CUDA;
  // No current context (a thread's first call) or another one than the attributes were
  // set in: set them again; cudaFuncSetAttribute makes the primary context current.
  const CUcontext ctx = current_ctx();
  std::lock_guard<std::mutex> lk(g_mu);
  DevInfo& d = g_dev[dev];
  if (!ctx || d.ctx != ctx) d.attrs_set = false;
  if (d.sms == 0) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return LORA_ERR_CUDA;
  }
  if (!d.attrs_set) {
    bool ok = true;
#define SET_SMEM(fn, bytes) ok &= cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess
    SET_SMEM((lora_gemm_pair_kernel<false, EPI_STORE>), (PairCfg<false>::SMEM_BYTES));
    SET_SMEM((lora_gemm_pair_kernel<true, EPI_STORE>), (PairCfg<true>::SMEM_BYTES));
    SET_SMEM((lora_gemm_pair_kernel<false, EPI_SWIGLU_FWD>), (PairCfg<false>::SMEM_BYTES));
    SET_SMEM((lora_gemm_pair_kernel<true, EPI_SWIGLU_BWD>), (PairCfg<true>::SMEM_BYTES));
#define SET_GEMM_Q(WF)                                                                              \
  SET_SMEM((lora_gemm_q_kernel<false, WF, EPI_STORE>), (QCfg<false, WF>::SMEM_BYTES));             \
  SET_SMEM((lora_gemm_q_kernel<true, WF, EPI_STORE>), (QCfg<true, WF>::SMEM_BYTES));               \
  SET_SMEM((lora_gemm_q_kernel<false, WF, EPI_SWIGLU_FWD>), (QCfg<false, WF>::SMEM_BYTES));        \
  SET_SMEM((lora_gemm_q_kernel<true, WF, EPI_SWIGLU_BWD>), (QCfg<true, WF>::SMEM_BYTES));
    SET_GEMM_Q(WF_BLOCK4)
    SET_GEMM_Q(WF_INT8)
    SET_GEMM_Q(WF_FP8)
#undef SET_GEMM_Q
    SET_SMEM(dualproj_kernel<DP_BOTH>, dual_smem_bytes());
    SET_SMEM(dualproj_kernel<DP_ROWS>, dual_smem_bytes());
    SET_SMEM(dualproj_kernel<DP_COLS>, dual_smem_bytes());
    SET_SMEM((lora_gemm_pair_kernel<false, EPI_CE_LSE>), (PairCfg<false>::SMEM_BYTES));
    SET_SMEM((lora_gemm_pair_kernel<false, EPI_CE_DLOGITS>), (PairCfg<false>::SMEM_BYTES));
    SET_SMEM((lora_gemm_pair_kernel<true, EPI_ACC_F32>), (PairCfg<true>::SMEM_BYTES));
    SET_SMEM((rowproj_kernel<16, false>), (rowproj_smem_bytes<16, false>()));
    SET_SMEM((rowproj_kernel<32, false>), (rowproj_smem_bytes<32, false>()));
    SET_SMEM((rowproj_kernel<64, false>), (rowproj_smem_bytes<64, false>()));
    SET_SMEM((rowproj_kernel<128, false>), (rowproj_smem_bytes<128, false>()));
    SET_SMEM((rowproj_kernel<16, true>), (rowproj_smem_bytes<16, true>()));
    SET_SMEM((rowproj_kernel<32, true>), (rowproj_smem_bytes<32, true>()));
    SET_SMEM((rowproj_kernel<64, true>), (rowproj_smem_bytes<64, true>()));
    SET_SMEM((rowproj_kernel<128, true>), (rowproj_smem_bytes<128, true>()));
    SET_SMEM((colproj_kernel<16>), (colproj_smem_bytes<16>()));
    SET_SMEM((colproj_kernel<32>), (colproj_smem_bytes<32>()));
    SET_SMEM((colproj_kernel<64>), (colproj_smem_bytes<64>()));
    SET_SMEM((colproj_kernel<128>), (colproj_smem_bytes<128>()));
    SET_SMEM(tcproj_kernel<TP_ROWS_K>, tcproj_smem_bytes());
    SET_SMEM(tcproj_kernel<TP_ROWS_MN>, tcproj_smem_bytes());
    SET_SMEM(tcproj_kernel<TP_COLS>, tcproj_smem_bytes());
#undef SET_SMEM
    if (!ok) return LORA_ERR_CUDA;
    d.ctx = current_ctx();
    if (!d.ctx) return LORA_ERR_CUDA;
    d.attrs_set = true;
  }
  *out = &d;
  return LORA_OK;
}

// ---------------------------------------------------------------- TMA descriptors
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

lora_status_t get_encode() {
  static std::once_flag once;
  static bool ok = false;
  std::call_once(once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess && fn) {
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
      ok = true;
    }
  });
  return ok ? LORA_OK : LORA_ERR_CUDA;
}

// Row-major [rows][inner] matrix with row pitch = inner * elem bytes.
// pitch_elems = 0: rows are packed (pitch = inner).
lora_status_t tmap_2d(CUtensorMap* m, CUtensorMapDataType dt, int elem_bytes, const void* base, uint64_t inner,
                      uint64_t rows, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw,
                      uint64_t pitch_elems = 0) {
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {(pitch_elems ? pitch_elems : inner) * static_cast<uint64_t>(elem_bytes)};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? LORA_OK : LORA_ERR_CUDA;
}
lora_status_t tmap_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t bi, uint32_t br) {
  return tmap_2d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, inner, rows, bi, br, CU_TENSOR_MAP_SWIZZLE_128B);
}

// ---------------------------------------------------------------- validation
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

lora_status_t check_weight(const lora_weight_t* W) {
  if (!W) return LORA_ERR_INVALID_ARG;
  if (W->fmt < LORA_W_BF16 || W->fmt > LORA_W_FP8_E4M3) return LORA_ERR_INVALID_ARG;
  if (W->reserved != 0) return LORA_ERR_INVALID_ARG;
  if (W->N <= 0 || W->K <= 0) return LORA_ERR_INVALID_ARG;
  if (W->N > (1LL << 30) || W->K > (1LL << 30)) return LORA_ERR_UNSUPPORTED;
  if (!W->data) return LORA_ERR_INVALID_ARG;
  if (!aligned16(W->data)) return LORA_ERR_ALIGNMENT;
  if (W->N % 8 != 0) return LORA_ERR_UNSUPPORTED;
  if (W->fmt == LORA_W_BF16) {
    if (W->K % 8 != 0) return LORA_ERR_UNSUPPORTED;
  } else if (W->fmt == LORA_W_BLOCK4) {
    if (W->K % 64 != 0) return LORA_ERR_UNSUPPORTED;
    if (!W->absmax || !W->codebook) return LORA_ERR_INVALID_ARG;
    if (!aligned16(W->absmax) || !aligned16(W->codebook)) return LORA_ERR_ALIGNMENT;
  } else {
    if (W->K % 16 != 0) return LORA_ERR_UNSUPPORTED;
    if (!W->absmax) return LORA_ERR_INVALID_ARG;
    if (!aligned16(W->absmax)) return LORA_ERR_ALIGNMENT;
  }
  return LORA_OK;
}

lora_status_t check_rank(int r, float s) {
  if (!std::isfinite(s)) return LORA_ERR_INVALID_ARG;
  if (r < 8 || r > 128 || r % 8 != 0) return LORA_ERR_UNSUPPORTED;
  return LORA_OK;
}

lora_status_t check_ptr(const void* p) {
  if (!p) return LORA_ERR_INVALID_ARG;
  if (!aligned16(p)) return LORA_ERR_ALIGNMENT;
  return LORA_OK;
}

#define TRY(x)                              \
  do {                                      \
    const lora_status_t _st = (x);          \
    if (_st != LORA_OK) return _st;         \
  } while (0)

lora_status_t last_launch() { return cudaGetLastError() == cudaSuccess ? LORA_OK : LORA_ERR_CUDA; }

int finalize_grid(size_t n) {
  const size_t g = (n + 255) / 256;
  return static_cast<int>(g < 4096 ? (g > 0 ? g : 1) : 4096);
}

// ---------------------------------------------------------------- skinny launches
template <bool Q_T>
lora_status_t launch_rowproj(const __nv_bfloat16* P, int ldp, const __nv_bfloat16* Q, float* part, int M, int Kred,
                             int r, Split sp, cudaStream_t st) {
  const dim3 grid(cdiv(M, SK_BM), sp.splits);
  const int tps = sp.tiles_per_split;
  if (r <= 16)
    launch_k(rowproj_kernel<16, Q_T>, grid, dim3(SK_THREADS), rowproj_smem_bytes<16, Q_T>(), st, P, ldp, Q, part, M,
             Kred, r, tps);
  else if (r <= 32)
    launch_k(rowproj_kernel<32, Q_T>, grid, dim3(SK_THREADS), rowproj_smem_bytes<32, Q_T>(), st, P, ldp, Q, part, M,
             Kred, r, tps);
  else if (r <= 64)
    launch_k(rowproj_kernel<64, Q_T>, grid, dim3(SK_THREADS), rowproj_smem_bytes<64, Q_T>(), st, P, ldp, Q, part, M,
             Kred, r, tps);
  else
    launch_k(rowproj_kernel<128, Q_T>, grid, dim3(SK_THREADS), rowproj_smem_bytes<128, Q_T>(), st, P, ldp, Q, part, M,
             Kred, r, tps);
  count_launch();
  return last_launch();
}

lora_status_t launch_colproj(const __nv_bfloat16* P, int ldp, const __nv_bfloat16* R, int ldr, float* part, int M,
                             int Kout, int r, Split sp, cudaStream_t st) {
  const dim3 grid(cdiv(Kout, SK_BM), sp.splits);
  const int tps = sp.tiles_per_split;
  if (r <= 16)
    launch_k(colproj_kernel<16>, grid, dim3(SK_THREADS), colproj_smem_bytes<16>(), st, P, ldp, R, ldr, part, M, Kout,
             r, tps);
  else if (r <= 32)
    launch_k(colproj_kernel<32>, grid, dim3(SK_THREADS), colproj_smem_bytes<32>(), st, P, ldp, R, ldr, part, M, Kout,
             r, tps);
  else if (r <= 64)
    launch_k(colproj_kernel<64>, grid, dim3(SK_THREADS), colproj_smem_bytes<64>(), st, P, ldp, R, ldr, part, M, Kout,
             r, tps);
  else
    launch_k(colproj_kernel<128>, grid, dim3(SK_THREADS), colproj_smem_bytes<128>(), st, P, ldp, R, ldr, part, M, Kout,
             r, tps);
  count_launch();
  return last_launch();
}

// partT [d.b][M][r] = P·Q summed per column block, partD [d.a][C][r] = Pᵀ·R summed per row
// block, for P [M][C] with row pitch ldp, Q = B [C][r] (DP_ROWS: Q = Aᵀ with A [r][C] as
// stored) and R with row pitch ldr; a single-product mode leaves the other partials alone.
template <int MODE>
lora_status_t launch_dual(const __nv_bfloat16* P, long long ldp, const __nv_bfloat16* Q, const __nv_bfloat16* R,
                          long long ldr, long long M, long long C, int r, const DualSplit& d, float* partT,
                          float* partD, uint32_t* status, cudaStream_t st) {
  CUtensorMap tp, tq, tr;
  TRY(tmap_2d(&tp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, P, C, M, 64, DP_TR, CU_TENSOR_MAP_SWIZZLE_128B, ldp));
  if (MODE == DP_ROWS)
    TRY(tmap_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Q, C, r, DP_TC, DP_RPAD, CU_TENSOR_MAP_SWIZZLE_NONE));
  else if (MODE == DP_BOTH)
    TRY(tmap_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Q, r, C, DP_RPAD, DP_TC, CU_TENSOR_MAP_SWIZZLE_NONE));
  else
    tq = tp;  // not read
  if (MODE != DP_ROWS)
    TRY(tmap_2d(&tr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, R, r, M, DP_RPAD, DP_TR, CU_TENSOR_MAP_SWIZZLE_32B, ldr));
  else
    tr = tp;  // not read
  const DualParams dp{partT, partD, static_cast<int>(M), static_cast<int>(C), r, d.row_tiles, d.col_tiles, status,
                      wait_limit_ns()};
  launch_k(dualproj_kernel<MODE>, dim3(d.a, d.b), dim3(DP_THREADS), dual_smem_bytes(), st, tp, tq, tr, dp);
  count_launch();
  return last_launch();
}

// Tensor-core rank-r pass (tcproj.cuh).  Row projection: P [rows][red] with row pitch ldp
// and Q = A [r][red] (TP_ROWS_K) or B [red][r] with row pitch ldq (TP_ROWS_MN).  Column
// projection (TP_COLS): P [red][rows] with row pitch ldp and R [red][r] with row pitch ldq.
// Writes part [splits][rows][r].
template <int MODE>
lora_status_t launch_tcproj(const __nv_bfloat16* P, long long ldp, const __nv_bfloat16* Q, long long ldq,
                            long long rows, long long red, int r, const TcSplit& t, float* part, uint32_t* status,
                            cudaStream_t st) {
  const int rpad = r <= 64 ? 64 : 128;
  CUtensorMap tp, tq;
  if (MODE == TP_COLS) {
    TRY(tmap_2d(&tp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, P, rows, red, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B, ldp));
  } else {
    TRY(tmap_2d(&tp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, P, red, rows, 64, TP_BM, CU_TENSOR_MAP_SWIZZLE_128B, ldp));
  }
  if (MODE == TP_ROWS_K)
    TRY(tmap_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Q, red, r, 64, rpad, CU_TENSOR_MAP_SWIZZLE_128B, ldq));
  else
    TRY(tmap_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Q, r, red, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B, ldq));
  const TcProjParams tpp{part, static_cast<int>(rows), static_cast<int>(red), r, rpad, t.splits, t.fps, status,
                         wait_limit_ns()};
  launch_k(tcproj_kernel<MODE>, dim3(t.tiles * t.splits), dim3(TP_THREADS), tcproj_smem_bytes(), st, tp, tq, tpp);
  count_launch();
  return last_launch();
}

// Σ of the split partials [splits][rows][r] -> out1 (plain) and/or out2 (times scale),
// row i written at out + i*opitch.
lora_status_t finalize_rows(const float* part, int splits, long long rows, int r, int opitch, float scale,
                            __nv_bfloat16* out1, __nv_bfloat16* out2, cudaStream_t st) {
  const size_t n = static_cast<size_t>(rows) * r;
  launch_k(finalize_rows_kernel, dim3(finalize_grid(n / 2)), dim3(256), 0, st, part, splits, n, r, opitch, scale, out1, out2);
  count_launch();
  return last_launch();
}

// scale · Σ of the split partials [splits][C][r] -> out [C][r], or [r][C] if transpose;
// out is bf16, or fp32 when f32 (adapter gradients summed over ranks before rounding).
lora_status_t finalize_cols(const float* part, int splits, int C, int r, float scale, bool transpose, void* out,
                            bool f32, cudaStream_t st) {
  const size_t n = static_cast<size_t>(C) * r;
  if (f32)
    launch_k(finalize_cols_kernel<float>, dim3(finalize_grid(n)), dim3(256), 0, st, part, splits, C, r, scale,
             transpose ? 1 : 0, static_cast<float*>(out));
  else
    launch_k(finalize_cols_kernel<__nv_bfloat16>, dim3(finalize_grid(n)), dim3(256), 0, st, part, splits, C, r, scale,
             transpose ? 1 : 0, static_cast<__nv_bfloat16*>(out));
  count_launch();
  return last_launch();
}

// Byte pointer `elems` elements into an adapter-gradient array of bf16 or fp32 elements.
inline void* grad_at(void* base, size_t elems, bool f32) {
  return static_cast<uint8_t*>(base) + elems * (f32 ? 4 : 2);
}

// ---------------------------------------------------------------- GEMM launch
template <bool B_MN, int EPI>
lora_status_t launch_gemm(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& e, const CUtensorMap& f,
                          const PairParams& p, int sms, cudaStream_t st) {
  using C = PairCfg<B_MN>;
  const long long tiles = static_cast<long long>(cdiv(p.M, C::BM)) * cdiv(p.Nout, EpiTile<EPI>::COLS);
  const long long pairs = p.sk_on ? kGemmPairs : (tiles < sms / 2 ? tiles : sms / 2);
  const int grid = static_cast<int>(2 * (pairs > 0 ? pairs : 1));
  {
    TimedRegion tr(B_MN ? LORA_KERNEL_BWD_GEMM : LORA_KERNEL_FWD_GEMM, st);
    launch_k(lora_gemm_pair_kernel<B_MN, EPI>, dim3(grid), dim3(C::template threads<EPI>()), C::SMEM_BYTES, st, a, b,
             e, f, p);
  }
  count_launch();
  return last_launch();
}

// Tensor-map boxes of the GEMM operands: 64 elements wide, 128 rows high (the quantized
// kernel's code and backward-F boxes are set in launch_gemm_w).
constexpr uint32_t kBoxX = 64, kBoxY = 128;

// The weight operand's tensor map (over the stored [N, K] array, for either direction)
// and the launch of the GEMM instantiation for the weight's format.
template <bool B_MN, int WF, int EPI>
lora_status_t launch_gemm_q(const CUtensorMap& a, const CUtensorMap& e, const CUtensorMap& f, const PairParams& p,
                            int sms, cudaStream_t st) {
  using C = QCfg<B_MN, WF>;
  const long long tiles = static_cast<long long>(cdiv(p.M, C::BM)) * cdiv(p.Nout, EpiTile<EPI>::COLS);
  const long long pairs = p.sk_on ? kGemmPairs : (tiles < sms / 2 ? tiles : sms / 2);
  const int grid = static_cast<int>(2 * (pairs > 0 ? pairs : 1));
  // the raster group counts tiles; 512-row tiles take half as many for the same rows
  PairParams q = p;
  q.group_m = p.group_m > 1 ? p.group_m / 2 : 1;
  // the staged store epilogue's output map: 32 × 32 boxes, 64-byte swizzle
  CUtensorMap o = a;  // not read by the other epilogues
  if (EPI == EPI_STORE && C::STAGED_STORE)
    TRY(tmap_2d(&o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.out, p.Nout, p.M, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B));
  {
    TimedRegion tr(B_MN ? LORA_KERNEL_BWD_GEMM : LORA_KERNEL_FWD_GEMM, st);
    launch_k(lora_gemm_q_kernel<B_MN, WF, EPI>, dim3(grid), dim3(C::NUM_THREADS), C::SMEM_BYTES, st, a, e, f, o, q);
  }
  count_launch();
  return last_launch();
}

// The LoRA F operand: its array and shape; its tensor map's box depends on the kernel.
struct FSpec {
  const void* base;
  uint64_t inner, rows;
};

// The weight operand's tensor map (over the stored [N, K] array, for either direction)
// and the launch of the GEMM for the weight's format: the bf16 pair kernel, or the
// quantized kernel, whose fills are 64 deep.
template <bool B_MN, int EPI>
lora_status_t launch_gemm_w(const lora_weight_t* W, const CUtensorMap& a, const CUtensorMap& e, const FSpec& fs,
                            const PairParams& p, int sms, cudaStream_t st) {
  CUtensorMap b, f;
  TRY(tmap_bf16(&f, fs.base, fs.inner, fs.rows, kBoxX, kBoxY));
  if constexpr (EPI == EPI_CE_LSE || EPI == EPI_CE_DLOGITS || EPI == EPI_ACC_F32) {
    // the cross-entropy head is bf16 only (checked by the caller)
    TRY(tmap_bf16(&b, W->data, W->K, W->N, kBoxX, kBoxY));
    return launch_gemm<B_MN, EPI>(a, b, e, f, p, sms, st);
  } else {
    if (W->fmt == LORA_W_BF16) {
      TRY(tmap_bf16(&b, W->data, W->K, W->N, kBoxX, kBoxY));
      return launch_gemm<B_MN, EPI>(a, b, e, f, p, sms, st);
    }
    // the quantized kernel's backward LoRA fill takes 64 ranks per box; its dequant
    // threads load the codes themselves (PairParams::codes)
    if (B_MN) TRY(tmap_bf16(&f, fs.base, fs.inner, fs.rows, kBoxX, 64));
    switch (W->fmt) {
      case LORA_W_BLOCK4: return launch_gemm_q<B_MN, WF_BLOCK4, EPI>(a, e, f, p, sms, st);
      case LORA_W_INT8: return launch_gemm_q<B_MN, WF_INT8, EPI>(a, e, f, p, sms, st);
      default: return launch_gemm_q<B_MN, WF_FP8, EPI>(a, e, f, p, sms, st);
    }
  }
}

// ---------------------------------------------------------------- output segments
// Grouped projections share X: W, A and B stack the projections' weights, adapters
// A_g [r, K] and B_g [N_g, r] along rows.  A single projection is one segment.
struct Segs {
  int n = 1;
  long long rows[LORA_MAX_SEGMENTS] = {};
  long long off[LORA_MAX_SEGMENTS + 1] = {};
};

lora_status_t make_segs(const lora_segments_t* sg, long long N, Segs* out) {
  Segs s;
  if (!sg) {
    s.n = 1;
    s.rows[0] = N;
    s.off[1] = N;
    *out = s;
    return LORA_OK;
  }
  if (sg->count < 1 || sg->count > LORA_MAX_SEGMENTS || sg->reserved != 0) return LORA_ERR_INVALID_ARG;
  s.n = sg->count;
  for (int g = 0; g < s.n; ++g) {
    if (sg->rows[g] <= 0) return LORA_ERR_INVALID_ARG;
    if (sg->rows[g] % 8 != 0) return LORA_ERR_UNSUPPORTED;
    s.rows[g] = sg->rows[g];
    s.off[g + 1] = s.off[g] + sg->rows[g];
    // a 256-column output tile must not straddle two projections
    if (g + 1 < s.n && s.off[g + 1] % 256 != 0) return LORA_ERR_UNSUPPORTED;
  }
  if (s.off[s.n] != N) return LORA_ERR_INVALID_ARG;
  *out = s;
  return LORA_OK;
}

void set_segments(PairParams& p, const Segs& sg, int e_stride) {
  p.nseg = sg.n;
  p.e_seg_stride = e_stride;
  for (int g = 0; g < LORA_MAX_SEGMENTS; ++g)
    p.seg_end_tile[g] = g < sg.n ? static_cast<int>(sg.off[g + 1] / 256) : 0x7fffffff;
}

PairParams gemm_params(long long M, long long Nout, long long Kred, int r, void* out, uint32_t* status,
                       const lora_weight_t* W) {
  PairParams p{};
  p.M = static_cast<int>(M);
  p.Nout = static_cast<int>(Nout);
  p.Kred = static_cast<int>(Kred);
  p.r = r;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.sk_on = 0;
  p.sk_dp_tiles = 0;
  p.kpart = nullptr;
  p.status = status;
  p.wait_ns = wait_limit_ns();
  p.group_m = group_m_default();
  p.nseg = 1;
  p.e_seg_stride = 0;
  for (int g = 0; g < LORA_MAX_SEGMENTS; ++g) p.seg_end_tile[g] = 0x7fffffff;
  p.Nw = static_cast<int>(W->N);
  p.Kw = static_cast<int>(W->K);
  p.codes = W->fmt != LORA_W_BF16 ? static_cast<const uint8_t*>(W->data) : nullptr;
  if (W->fmt == LORA_W_BLOCK4) {
    p.absmax = static_cast<const __half*>(W->absmax);
    p.codebook = W->codebook;
  } else if (W->fmt != LORA_W_BF16) {
    p.row_scale = static_cast<const float*>(W->absmax);
  }
  return p;
}

// The stream-K schedule for the plain store epilogue when the sizes call for it, the GPU
// runs the 74 CTA pairs it is planned for, and its slots fit in the caller's part region
// (callers without room keep whole tiles).
GemmSched set_sched(PairParams& p, const lora_weight_t* W, float* part, size_t part_cap, int sms) {
  const bool q = W->fmt != LORA_W_BF16;
  GemmSched g = gemm_sched(p.M, p.Nout, p.Kred, p.r, q);
  if (g.sk && part && sms / 2 >= kGemmPairs && gemm_sched_bytes(p.M, p.Nout, p.Kred, p.r, q) <= part_cap) {
    p.sk_on = 1;
    p.sk_dp_tiles = g.dp_tiles;
    p.kpart = part;
  } else {
    g.sk = false;
  }
  return g;
}

// The tiles stream-K cut into pieces: out = Σ of their slots in pair order.
lora_status_t streamk_fixup(const PairParams& p, const GemmSched& g, cudaStream_t st) {
  if (!g.sk) return LORA_OK;
  const int num_m = cdiv(p.M, g.tile_rows), num_n = cdiv(p.Nout, 256);
  const int group_m = g.tile_rows == 512 ? (p.group_m > 1 ? p.group_m / 2 : 1) : p.group_m;
  const dim3 grid(kGemmPairs - 1, g.tile_rows / 8);  // 8 tile rows per block
  if (g.tile_rows == 512)
    launch_k(streamk_fixup_kernel<512>, grid, dim3(256), 0, st, p.kpart, p.out, p.M, p.Nout, num_m, num_n, group_m,
             g.dp_tiles, num_m * num_n, g.tile_fills, kGemmPairs);
  else
    launch_k(streamk_fixup_kernel<256>, grid, dim3(256), 0, st, p.kpart, p.out, p.M, p.Nout, num_m, num_n, group_m,
             g.dp_tiles, num_m * num_n, g.tile_fills, kGemmPairs);
  count_launch();
  return last_launch();
}

// ---------------------------------------------------------------- forward core
// XA = X·Aᵀ for all segments at once (rank G·r), then Y = X·Wᵀ + s·XA_g·B_gᵀ with the
// LoRA fill of each output tile taking its segment's columns of s·XA.
lora_status_t forward_core(const void* X, long long M, const lora_weight_t* W, const Segs& sg, const void* A,
                           const void* B, int r, float s, void* Y, void* XA, __nv_bfloat16* sXA, float* part,
                           size_t part_cap, uint32_t* status, cudaStream_t st) {
  DevInfo* dev = nullptr;
  TRY(dev_info(&dev));
  TRY(get_encode());
  const long long N = W->N, K = W->K;
  const int rt = sg.n * r;
  const int Mi = static_cast<int>(M), Ki = static_cast<int>(K);
  const auto* Xb = static_cast<const __nv_bfloat16*>(X);

  const DualSplit ds = dual_split(M, K, rt, DP_ROWS);
  if (tc_rank(rt) && tc_part_bytes(M, K, rt) <= part_cap) {
    // X·Aᵀ on the tensor cores
    const TcSplit t = tc_split(M, K, rt);
    TRY(launch_tcproj<TP_ROWS_K>(Xb, K, static_cast<const __nv_bfloat16*>(A), K, M, K, rt, t, part, status, st));
    TRY(finalize_rows(part, t.splits, M, rt, rt, s, static_cast<__nv_bfloat16*>(XA), sXA, st));
  } else if (ds.use && dual_part_t_bytes(ds, M, rt) <= part_cap) {
    // one TMA-fed pass over X
    TRY(launch_dual<DP_ROWS>(Xb, K, static_cast<const __nv_bfloat16*>(A), nullptr, 0, M, K, rt, ds, part, nullptr,
                             status, st));
    TRY(finalize_rows(part, ds.b, M, rt, rt, s, static_cast<__nv_bfloat16*>(XA), sXA, st));
  } else {
    const Split sp = rowproj_split(M, K);
    TRY(launch_rowproj<false>(Xb, Ki, static_cast<const __nv_bfloat16*>(A), part, Mi, Ki, rt, sp, st));
    TRY(finalize_rows(part, sp.splits, M, rt, rt, s, static_cast<__nv_bfloat16*>(XA), sXA, st));
  }

  CUtensorMap ta, te;
  TRY(tmap_bf16(&ta, X, K, M, kBoxX, kBoxY));
  TRY(tmap_bf16(&te, sXA, rt, M, kBoxX, kBoxY));
  const FSpec tf{B, static_cast<uint64_t>(r), static_cast<uint64_t>(N)};
  PairParams p = gemm_params(M, N, K, r, Y, status, W);
  set_segments(p, sg, r);
  const GemmSched g = set_sched(p, W, part, part_cap, dev->sms);
  TRY((launch_gemm_w<false, EPI_STORE>(W, ta, te, tf, p, dev->sms, st)));
  return streamk_fixup(p, g, st);
}

// ---------------------------------------------------------------- backward core
lora_status_t backward_core(const void* dY, const void* X, const void* XA, long long M, const lora_weight_t* W,
                            const Segs& sg, const void* A, const void* B, int r, float s, void* dX, void* dA,
                            void* dB, bool f32, __nv_bfloat16* sdYB, float* part, size_t part_cap, uint32_t* status,
                            cudaStream_t st) {
  DevInfo* dev = nullptr;
  TRY(dev_info(&dev));
  TRY(get_encode());
  const long long N = W->N, K = W->K;
  const int rt = sg.n * r;
  const int Mi = static_cast<int>(M), Ni = static_cast<int>(N), Ki = static_cast<int>(K);
  const auto* dYb = static_cast<const __nv_bfloat16*>(dY);
  const auto* Xb = static_cast<const __nv_bfloat16*>(X);
  const auto* Bb = static_cast<const __nv_bfloat16*>(B);
  const auto* XAb = static_cast<const __nv_bfloat16*>(XA);

  for (int g = 0; g < sg.n; ++g) {
    const int rows = static_cast<int>(sg.rows[g]);
    const long long o = sg.off[g];
    void* dBg = grad_at(dB, static_cast<size_t>(o) * r, f32);
    const DualSplit ds = dual_split(M, rows, r);
    if (tc_rank(r) && tc_part_bytes(M, rows, r) <= part_cap && tc_part_bytes(rows, M, r) <= part_cap) {
      // s·dY_g·B_g and dB_g = s·dY_gᵀ·XA_g on the tensor cores, one pass each
      TcSplit t = tc_split(M, rows, r);
      TRY(launch_tcproj<TP_ROWS_MN>(dYb + o, N, Bb + o * r, r, M, rows, r, t, part, status, st));
      TRY(finalize_rows(part, t.splits, M, r, rt, s, nullptr, sdYB + g * r, st));
      t = tc_split(rows, M, r);
      TRY(launch_tcproj<TP_COLS>(dYb + o, N, XAb + g * r, rt, rows, M, r, t, part, status, st));
      TRY(finalize_cols(part, t.splits, rows, r, s, false, dBg, f32, st));
      continue;
    }
    if (ds.use && dual_part_bytes(ds, M, rows, r) <= part_cap) {
      // one pass over dY_g for s·dY_g·B_g (columns [g·r, g·r + r) of s·dY·B) and dB_g = s·dY_gᵀ·XA_g
      float* partD = part + dual_part_t_bytes(ds, M, r) / 4;
      TRY(launch_dual<DP_BOTH>(dYb + o, N, Bb + o * r, XAb + g * r, rt, M, rows, r, ds, part, partD, status, st));
      TRY(finalize_rows(part, ds.b, M, r, rt, s, nullptr, sdYB + g * r, st));
      TRY(finalize_cols(partD, ds.a, rows, r, s, false, dBg, f32, st));
      continue;
    }
    // s·dY_g·B_g -> columns [g·r, g·r + r) of s·dY·B
    Split sp = rowproj_split(M, rows);
    TRY(launch_rowproj<true>(dYb + o, Ni, Bb + o * r, part, Mi, rows, r, sp, st));
    TRY(finalize_rows(part, sp.splits, M, r, rt, s, nullptr, sdYB + g * r, st));
    // dB_g = s·dY_gᵀ·XA_g
    sp = colproj_split(M, rows);
    TRY(launch_colproj(dYb + o, Ni, XAb + g * r, rt, part, Mi, rows, r, sp, st));
    TRY(finalize_cols(part, sp.splits, rows, r, s, false, dBg, f32, st));
  }
  if (dX) {
    // dX = dY·W + (s·dY·B)·A with the LoRA fill over all G·r ranks
    CUtensorMap ta, te;
    TRY(tmap_bf16(&ta, dY, N, M, kBoxX, kBoxY));
    TRY(tmap_bf16(&te, sdYB, rt, M, kBoxX, kBoxY));
    const FSpec tf{A, static_cast<uint64_t>(K), static_cast<uint64_t>(rt)};
    PairParams p = gemm_params(M, K, N, rt, dX, status, W);
    const GemmSched g = set_sched(p, W, part, part_cap, dev->sms);
    TRY((launch_gemm_w<true, EPI_STORE>(W, ta, te, tf, p, dev->sms, st)));
    TRY(streamk_fixup(p, g, st));
  }
  // dA = (s·dY·B)ᵀ·X, computed as Xᵀ·(s·dY·B) and written transposed [G·r, K]
  if (tc_rank(rt) && tc_part_bytes(K, M, rt) <= part_cap) {
    const TcSplit t = tc_split(K, M, rt);
    TRY(launch_tcproj<TP_COLS>(Xb, K, sdYB, rt, K, M, rt, t, part, status, st));
    return finalize_cols(part, t.splits, Ki, rt, 1.0f, true, dA, f32, st);
  }
  const DualSplit dsa = dual_split(M, K, rt, DP_COLS);
  if (dsa.use && dual_part_d_bytes(dsa, K, rt) <= part_cap) {
    // one TMA-fed pass over X
    TRY(launch_dual<DP_COLS>(Xb, K, nullptr, sdYB, rt, M, K, rt, dsa, nullptr, part, status, st));
    return finalize_cols(part, dsa.a, Ki, rt, 1.0f, true, dA, f32, st);
  }
  const Split sp = colproj_split(M, K);
  TRY(launch_colproj(Xb, Ki, sdYB, rt, part, Mi, Ki, rt, sp, st));
  return finalize_cols(part, sp.splits, Ki, rt, 1.0f, true, dA, f32, st);
}

// ---------------------------------------------------------------- argument checks shared by the entries
lora_status_t check_common(const lora_weight_t* W, const lora_segments_t* segs, int r, float s, long long M,
                           const void* A, const void* B, Segs* sg) {
  TRY(check_weight(W));
  TRY(check_rank(r, s));
  if (M < 0 || M > (1LL << 31) - 256) return LORA_ERR_INVALID_ARG;
  TRY(make_segs(segs, W->N, sg));
  if (sg->n * r > 128) return LORA_ERR_UNSUPPORTED;
  TRY(check_ptr(A));
  TRY(check_ptr(B));
  return LORA_OK;
}

lora_status_t fwd_entry(const void* X, int64_t M, const lora_weight_t* W, const lora_segments_t* segs, const void* A,
                        const void* B, int32_t r, float s, void* Y, void* XA, void* workspace, size_t ws_bytes,
                        void* stream) {
  Segs sg;
  TRY(check_common(W, segs, r, s, M, A, B, &sg));
  if (M == 0) return LORA_OK;
  TRY(check_ptr(X));
  TRY(check_ptr(Y));
  TRY(check_ptr(XA));
  const WsLayout wl = ws_layout(M, W->N, W->K, r, sg.n, W->fmt != LORA_W_BF16);
  if (!workspace) return LORA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return LORA_ERR_ALIGNMENT;
  if (ws_bytes < wl.total) return LORA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  return forward_core(X, M, W, sg, A, B, r, s, Y, XA, reinterpret_cast<__nv_bfloat16*>(ws + wl.skinny_off),
                      reinterpret_cast<float*>(ws + wl.part_off), wl.total - wl.part_off,
                      reinterpret_cast<uint32_t*>(ws), static_cast<cudaStream_t>(stream));
}

lora_status_t bwd_entry(const void* dY, const void* X, const void* XA, int64_t M, const lora_weight_t* W,
                        const lora_segments_t* segs, const void* A, const void* B, int32_t r, float s, void* dX,
                        void* dA, void* dB, uint32_t flags, void* workspace, size_t ws_bytes, void* stream) {
  Segs sg;
  if (flags & ~static_cast<uint32_t>(LORA_GRADS_F32)) return LORA_ERR_INVALID_ARG;
  const bool f32 = (flags & LORA_GRADS_F32) != 0;
  TRY(check_common(W, segs, r, s, M, A, B, &sg));
  TRY(check_ptr(dA));
  TRY(check_ptr(dB));
  const long long N = W->N, K = W->K;
  const int rt = sg.n * r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t esz = f32 ? 4 : 2;
  if (M == 0) {
    if (cudaMemsetAsync(dA, 0, static_cast<size_t>(rt) * K * esz, st) != cudaSuccess) return LORA_ERR_CUDA;
    if (cudaMemsetAsync(dB, 0, static_cast<size_t>(N) * r * esz, st) != cudaSuccess) return LORA_ERR_CUDA;
    return LORA_OK;
  }
  TRY(check_ptr(dY));
  TRY(check_ptr(X));
  TRY(check_ptr(XA));
  if (dX && !aligned16(dX)) return LORA_ERR_ALIGNMENT;
  const WsLayout wl = ws_layout(M, N, K, r, sg.n, W->fmt != LORA_W_BF16);
  if (!workspace) return LORA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return LORA_ERR_ALIGNMENT;
  if (ws_bytes < wl.total) return LORA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  return backward_core(dY, X, XA, M, W, sg, A, B, r, s, dX, dA, dB, f32,
                       reinterpret_cast<__nv_bfloat16*>(ws + wl.skinny_off), reinterpret_cast<float*>(ws + wl.part_off),
                       wl.total - wl.part_off, reinterpret_cast<uint32_t*>(ws), st);
}

// ---------------------------------------------------------------- feed-forward block
// Workspace of the block: the status head, one bf16 skinny operand of rank 2r and the
// largest set of fp32 split partials any of its skinny passes needs.
WsLayout mlp_ws_layout(long long M, long long D, long long I, int r) {
  WsLayout w;
  w.skinny_off = kStatusBytes;
  w.part_off = w.skinny_off + align256(static_cast<size_t>(M) * 2 * r * 2);
  size_t part = 0;
  auto upd = [&](size_t b) { part = b > part ? b : part; };
  upd(static_cast<size_t>(rowproj_split(M, D).splits) * M * 2 * r * 4);  // [X·A_gᵀ | X·A_uᵀ]
  upd(static_cast<size_t>(rowproj_split(M, I).splits) * M * r * 4);      // H·A_dᵀ, dG·B_g, dU·B_u
  upd(static_cast<size_t>(rowproj_split(M, D).splits) * M * r * 4);      // dZ·B_d
  upd(static_cast<size_t>(colproj_split(M, D).splits) * D * r * 4);      // dB_d
  upd(static_cast<size_t>(colproj_split(M, I).splits) * I * r * 4);      // dA_d, dB_g, dB_u
  upd(static_cast<size_t>(colproj_split(M, D).splits) * D * 2 * r * 4);  // [dA_g; dA_u]
  upd(dual_part_bytes(dual_split(M, D, r), M, D, r));                    // dZ·B_d and dZᵀ·(H·A_dᵀ)
  upd(dual_part_bytes(dual_split(M, I, r), M, I, r));                    // dG·B_g and dGᵀ·XA_g (and the up half)
  if (tc_rank(2 * r)) {
    upd(tc_part_bytes(M, D, 2 * r));  // [X·A_gᵀ | X·A_uᵀ] on the tensor cores
    upd(tc_part_bytes(D, M, 2 * r));  // [dA_g; dA_u]
  }
  if (tc_rank(r)) {
    upd(tc_part_bytes(M, I, r));  // H·A_dᵀ, dG·B_g, dU·B_u
    upd(tc_part_bytes(I, M, r));  // dA_d, dB_g, dB_u
    upd(tc_part_bytes(M, D, r));  // dZ·B_d
    upd(tc_part_bytes(D, M, r));  // dB_d
  }
  w.total = w.part_off + align256(part);
  return w;
}

lora_status_t mlp_check(const lora_mlp_t* m, int r, float s, long long M) {
  if (!m) return LORA_ERR_INVALID_ARG;
  TRY(check_weight(&m->gate_up));
  TRY(check_weight(&m->down));
  if (m->gate_up.fmt != m->down.fmt) return LORA_ERR_INVALID_ARG;
  TRY(check_rank(r, s));
  if (2 * r > 128) return LORA_ERR_UNSUPPORTED;
  if (M < 0 || M > (1LL << 31) - 256) return LORA_ERR_INVALID_ARG;
  const long long D = m->gate_up.K, I = m->down.K;
  if (m->gate_up.N != 2 * I || m->down.N != D) return LORA_ERR_INVALID_ARG;
  TRY(check_ptr(m->A_gate_up));
  TRY(check_ptr(m->B_gate_up));
  TRY(check_ptr(m->A_down));
  TRY(check_ptr(m->B_down));
  return LORA_OK;
}

Segs gate_up_segs(long long I) {
  Segs g;
  g.n = 2;
  g.rows[0] = g.rows[1] = I;
  g.off[1] = I;
  g.off[2] = 2 * I;
  return g;
}

// [X·A_gᵀ | X·A_uᵀ] in one pass over X; one GEMM for gate and up whose epilogue writes
// G, U and H = silu(G)·U; then the down projection as a LoRA linear of H.
lora_status_t mlp_forward_core(const void* X, long long M, const lora_mlp_t* m, int r, float s, void* Z, void* GU,
                               void* H, void* XAgu, void* XAd, __nv_bfloat16* skinny, float* part, size_t part_cap,
                               uint32_t* status, cudaStream_t st) {
  DevInfo* dev = nullptr;
  TRY(dev_info(&dev));
  TRY(get_encode());
  const long long D = m->gate_up.K, I = m->down.K;
  const int r2 = 2 * r;
  const int Mi = static_cast<int>(M), Di = static_cast<int>(D);
  if (tc_rank(r2) && tc_part_bytes(M, D, r2) <= part_cap) {
    const TcSplit t = tc_split(M, D, r2);
    TRY(launch_tcproj<TP_ROWS_K>(static_cast<const __nv_bfloat16*>(X), D,
                                 static_cast<const __nv_bfloat16*>(m->A_gate_up), D, M, D, r2, t, part, status, st));
    TRY(finalize_rows(part, t.splits, M, r2, r2, s, static_cast<__nv_bfloat16*>(XAgu), skinny, st));
  } else {
    const Split sp = rowproj_split(M, D);
    TRY(launch_rowproj<false>(static_cast<const __nv_bfloat16*>(X), Di,
                              static_cast<const __nv_bfloat16*>(m->A_gate_up), part, Mi, Di, r2, sp, st));
    TRY(finalize_rows(part, sp.splits, M, r2, r2, s, static_cast<__nv_bfloat16*>(XAgu), skinny, st));
  }

  CUtensorMap ta, te;
  TRY(tmap_bf16(&ta, X, D, M, kBoxX, kBoxY));
  TRY(tmap_bf16(&te, skinny, r2, M, kBoxX, kBoxY));
  const FSpec tf{m->B_gate_up, static_cast<uint64_t>(r), static_cast<uint64_t>(2 * I)};
  PairParams p = gemm_params(M, I, D, r2, H, status, &m->gate_up);
  p.half_rows = static_cast<int>(I);
  p.f_shift = r;
  p.aux = static_cast<__nv_bfloat16*>(GU);
  p.ld_aux = static_cast<int>(2 * I);
  p.aux_off = static_cast<int>(I);
  TRY((launch_gemm_w<false, EPI_SWIGLU_FWD>(&m->gate_up, ta, te, tf, p, dev->sms, st)));
  Segs one;
  one.rows[0] = D;
  one.off[1] = D;
  return forward_core(H, M, &m->down, one, m->A_down, m->B_down, r, s, Z, XAd, skinny, part, part_cap, status, st);
}

// Down projection's backward with SwiGLU's derivative in the dH GEMM's epilogue (GU
// becomes [dG | dU]), then gate and up as two projections of X with dY = [dG | dU].
lora_status_t mlp_backward_core(const void* dZ, const void* X, void* GU, const void* H, const void* XAgu,
                                const void* XAd, long long M, const lora_mlp_t* m, int r, float s, void* dX,
                                void* dAgu, void* dBgu, void* dAd, void* dBd, bool f32, __nv_bfloat16* skinny,
                                float* part, size_t part_cap, uint32_t* status, cudaStream_t st) {
  DevInfo* dev = nullptr;
  TRY(dev_info(&dev));
  TRY(get_encode());
  const long long D = m->gate_up.K, I = m->down.K;
  const int Mi = static_cast<int>(M), Di = static_cast<int>(D), Ii = static_cast<int>(I);
  const auto* dZb = static_cast<const __nv_bfloat16*>(dZ);
  const auto* Bd = static_cast<const __nv_bfloat16*>(m->B_down);
  const auto* XAdb = static_cast<const __nv_bfloat16*>(XAd);
  Split sp;
  const DualSplit ds = dual_split(M, D, r);
  if (ds.use && dual_part_bytes(ds, M, D, r) <= part_cap) {
    // one pass over dZ for s·dZ·B_d and dB_d = s·dZᵀ·(H·A_dᵀ)
    float* partD = part + dual_part_t_bytes(ds, M, r) / 4;
    TRY(launch_dual<DP_BOTH>(dZb, D, Bd, XAdb, r, M, D, r, ds, part, partD, status, st));
    TRY(finalize_rows(part, ds.b, M, r, r, s, nullptr, skinny, st));
    TRY(finalize_cols(partD, ds.a, Di, r, s, false, dBd, f32, st));
  } else if (tc_rank(r) && tc_part_bytes(M, D, r) <= part_cap && tc_part_bytes(D, M, r) <= part_cap) {
    // s·dZ·B_d and dB_d = s·dZᵀ·(H·A_dᵀ) on the tensor cores
    TcSplit t = tc_split(M, D, r);
    TRY(launch_tcproj<TP_ROWS_MN>(dZb, D, Bd, r, M, D, r, t, part, status, st));
    TRY(finalize_rows(part, t.splits, M, r, r, s, nullptr, skinny, st));
    t = tc_split(D, M, r);
    TRY(launch_tcproj<TP_COLS>(dZb, D, XAdb, r, D, M, r, t, part, status, st));
    TRY(finalize_cols(part, t.splits, Di, r, s, false, dBd, f32, st));
  } else {
    // s·dZ·B_d
    sp = rowproj_split(M, D);
    TRY(launch_rowproj<true>(dZb, Di, Bd, part, Mi, Di, r, sp, st));
    TRY(finalize_rows(part, sp.splits, M, r, r, s, nullptr, skinny, st));
    // dB_d = s·dZᵀ·(H·A_dᵀ)
    sp = colproj_split(M, D);
    TRY(launch_colproj(dZb, Di, XAdb, r, part, Mi, Di, r, sp, st));
    TRY(finalize_cols(part, sp.splits, Di, r, s, false, dBd, f32, st));
  }
  // dH = dZ·W_d + (s·dZ·B_d)·A_d, consumed by the epilogue: GU <- [dG | dU]
  {
    CUtensorMap ta, te;
    TRY(tmap_bf16(&ta, dZ, D, M, kBoxX, kBoxY));
    TRY(tmap_bf16(&te, skinny, r, M, kBoxX, kBoxY));
    const FSpec tf{m->A_down, static_cast<uint64_t>(I), static_cast<uint64_t>(r)};
    PairParams p = gemm_params(M, I, D, r, nullptr, status, &m->down);
    p.aux = static_cast<__nv_bfloat16*>(GU);
    p.ld_aux = static_cast<int>(2 * I);
    p.aux_off = static_cast<int>(I);
    TRY((launch_gemm_w<true, EPI_SWIGLU_BWD>(&m->down, ta, te, tf, p, dev->sms, st)));
  }
  // dA_d = (s·dZ·B_d)ᵀ·H
  if (tc_rank(r) && tc_part_bytes(I, M, r) <= part_cap) {
    const TcSplit t = tc_split(I, M, r);
    TRY(launch_tcproj<TP_COLS>(static_cast<const __nv_bfloat16*>(H), I, skinny, r, I, M, r, t, part, status, st));
    TRY(finalize_cols(part, t.splits, Ii, r, 1.0f, true, dAd, f32, st));
  } else {
    sp = colproj_split(M, I);
    TRY(launch_colproj(static_cast<const __nv_bfloat16*>(H), Ii, skinny, r, part, Mi, Ii, r, sp, st));
    TRY(finalize_cols(part, sp.splits, Ii, r, 1.0f, true, dAd, f32, st));
  }
  return backward_core(GU, X, XAgu, M, &m->gate_up, gate_up_segs(I), m->A_gate_up, m->B_gate_up, r, s, dX, dAgu,
                       dBgu, f32, skinny, part, part_cap, status, st);
}

lora_status_t mlp_ws_check(long long M, const lora_mlp_t* m, int r, void* workspace, size_t ws_bytes) {
  const WsLayout wl = mlp_ws_layout(M, m->gate_up.K, m->down.K, r);
  if (!workspace) return LORA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return LORA_ERR_ALIGNMENT;
  if (ws_bytes < wl.total) return LORA_ERR_WORKSPACE;
  return LORA_OK;
}

// ---------------------------------------------------------------- cross-entropy over an LM head
// Workspace: status head, then for the forward the per-tile partials [ceil(V/256)][M][2]
// and the label logits [M]; for the backward (the same bytes, reused) an fp32 dX running
// sum [M, D] and one bf16 slice of dlogits [M, Vc].
struct CeLayout {
  size_t part_off, zy_off, fwd_total, acc_off, dlog_off, bwd_fixed;
};
CeLayout ce_layout(long long M, long long D, long long V) {
  CeLayout c;
  c.part_off = kStatusBytes;
  c.zy_off = c.part_off + align256(static_cast<size_t>(cdiv(V, 256)) * M * 8);
  c.fwd_total = c.zy_off + align256(static_cast<size_t>(M) * 4);
  c.acc_off = kStatusBytes;
  c.dlog_off = c.acc_off + align256(static_cast<size_t>(M) * D * 4);
  c.bwd_fixed = c.dlog_off;
  return c;
}

lora_status_t ce_check(const void* X, long long M, const lora_weight_t* W, const int32_t* labels) {
  TRY(check_weight(W));
  if (W->fmt != LORA_W_BF16) return LORA_ERR_UNSUPPORTED;
  if (M < 0 || M > (1LL << 31) - 256) return LORA_ERR_INVALID_ARG;
  if (W->N > (1LL << 31) - 256) return LORA_ERR_UNSUPPORTED;
  if (M == 0) return LORA_OK;
  TRY(check_ptr(X));
  TRY(check_ptr(labels));
  return LORA_OK;
}

PairParams ce_params(long long M, long long Nout, long long Kred, void* out, uint32_t* status,
                     const lora_weight_t* W) {
  PairParams p = gemm_params(M, Nout, Kred, 0, out, status, W);
  return p;
}

size_t workspace_bytes_for(int64_t M, int64_t N, int64_t K, int32_t r, int32_t nseg, int32_t fmt) {
  if (M < 0 || N <= 0 || K <= 0 || r < 8 || r > 128 || r % 8) return 0;
  if (nseg < 1 || nseg > LORA_MAX_SEGMENTS || nseg * r > 128) return 0;
  if (fmt < LORA_W_BF16 || fmt > LORA_W_FP8_E4M3) return 0;
  if (M > (1LL << 31) - 256 || N > (1LL << 30) || K > (1LL << 30)) return 0;
  return ws_layout(M, N, K, r, nseg, fmt != LORA_W_BF16).total;
}

}  // namespace
}  // namespace lora

using namespace lora;

extern "C" {

const char* lora_status_string(int32_t status) {
  switch (status) {
    case LORA_OK: return "ok";
    case LORA_ERR_INVALID_ARG: return "invalid argument (null pointer, bad size, non-finite scale or bad enum)";
    case LORA_ERR_ALIGNMENT: return "a device pointer is not 16-byte aligned";
    case LORA_ERR_UNSUPPORTED:
      return "unsupported sizes (need 8<=r<=128, r%8==0, N%8==0, K%8==0; K%64==0 for 4-bit; "
             "projections of a group start at multiples of 256 rows and G*r<=128)";
    case LORA_ERR_WORKSPACE: return "workspace missing or smaller than lora_workspace_bytes()";
    case LORA_ERR_CUDA: return "a CUDA call failed";
    case LORA_ERR_DEVICE_TIMEOUT: return "a kernel gave up a bounded wait; outputs of that call are undefined";
    case LORA_ERR_DEVICE_BOUNDS:
      return "checked build: a kernel found a tile or copy origin out of range and skipped it; outputs undefined";
    case LORA_ERR_SCRATCH_LIMIT:
      return "problem needs more scratch than the fixed LORA_NOALLOC_SCRATCH_BYTES of lora_linear_fwd_noalloc";
    default: return "unknown status";
  }
}

int32_t lora_version(void) { return 200; }

size_t lora_workspace_bytes(int64_t M, int64_t N, int64_t K, int32_t r, int32_t fmt) {
  return workspace_bytes_for(M, N, K, r, 1, fmt);
}

size_t lora_grouped_workspace_bytes(int64_t M, int64_t N, int64_t K, int32_t r, int32_t nseg, int32_t fmt) {
  return workspace_bytes_for(M, N, K, r, nseg, fmt);
}

lora_status_t lora_linear_fwd(const void* X, int64_t M, const lora_weight_t* W, const void* A, const void* B, int32_t r,
                              float s, void* Y, void* XA, void* workspace, size_t ws_bytes, void* stream) {
  return fwd_entry(X, M, W, nullptr, A, B, r, s, Y, XA, workspace, ws_bytes, stream);
}

lora_status_t lora_linear_bwd(const void* dY, const void* X, const void* XA, int64_t M, const lora_weight_t* W,
                              const void* A, const void* B, int32_t r, float s, void* dX, void* dA, void* dB,
                              void* workspace, size_t ws_bytes, void* stream) {
  return bwd_entry(dY, X, XA, M, W, nullptr, A, B, r, s, dX, dA, dB, 0u, workspace, ws_bytes, stream);
}

lora_status_t lora_linear_bwd_ex(const void* dY, const void* X, const void* XA, int64_t M, const lora_weight_t* W,
                                 const void* A, const void* B, int32_t r, float s, void* dX, void* dA, void* dB,
                                 uint32_t flags, void* workspace, size_t ws_bytes, void* stream) {
  return bwd_entry(dY, X, XA, M, W, nullptr, A, B, r, s, dX, dA, dB, flags, workspace, ws_bytes, stream);
}

lora_status_t lora_grouped_fwd(const void* X, int64_t M, const lora_weight_t* W, const lora_segments_t* segs,
                               const void* A, const void* B, int32_t r, float s, void* Y, void* XA, void* workspace,
                               size_t ws_bytes, void* stream) {
  if (!segs) return LORA_ERR_INVALID_ARG;
  return fwd_entry(X, M, W, segs, A, B, r, s, Y, XA, workspace, ws_bytes, stream);
}

lora_status_t lora_grouped_bwd(const void* dY, const void* X, const void* XA, int64_t M, const lora_weight_t* W,
                               const lora_segments_t* segs, const void* A, const void* B, int32_t r, float s,
                               void* dX, void* dA, void* dB, void* workspace, size_t ws_bytes, void* stream) {
  if (!segs) return LORA_ERR_INVALID_ARG;
  return bwd_entry(dY, X, XA, M, W, segs, A, B, r, s, dX, dA, dB, 0u, workspace, ws_bytes, stream);
}

lora_status_t lora_grouped_bwd_ex(const void* dY, const void* X, const void* XA, int64_t M, const lora_weight_t* W,
                                  const lora_segments_t* segs, const void* A, const void* B, int32_t r, float s,
                                  void* dX, void* dA, void* dB, uint32_t flags, void* workspace, size_t ws_bytes,
                                  void* stream) {
  if (!segs) return LORA_ERR_INVALID_ARG;
  return bwd_entry(dY, X, XA, M, W, segs, A, B, r, s, dX, dA, dB, flags, workspace, ws_bytes, stream);
}

lora_status_t lora_round_bf16(const float* src, void* dst, int64_t n, void* stream) {
  if (n < 0) return LORA_ERR_INVALID_ARG;
  if (n == 0) return LORA_OK;
  TRY(check_ptr(src));
  TRY(check_ptr(dst));
  {
    // the output may not overlap the input
    const uint8_t* a0 = reinterpret_cast<const uint8_t*>(src);
    const uint8_t* b0 = static_cast<const uint8_t*>(dst);
    if (b0 < a0 + static_cast<size_t>(n) * 4 && a0 < b0 + static_cast<size_t>(n) * 2) return LORA_ERR_INVALID_ARG;
  }
  DevInfo* dev = nullptr;
  TRY(dev_info(&dev));
  const size_t total = static_cast<size_t>(n);
  size_t grid = (total + 255) / 256;
  const size_t cap = static_cast<size_t>(dev->sms) * 8;
  if (grid > cap) grid = cap;
  launch_k(round_bf16_kernel, dim3(static_cast<int>(grid)), dim3(256), 0, static_cast<cudaStream_t>(stream), src,
           static_cast<__nv_bfloat16*>(dst), total);
  count_launch();
  return last_launch();
}

size_t lora_mlp_workspace_bytes(int64_t M, int64_t D, int64_t I, int32_t r, int32_t fmt) {
  if (M < 0 || D <= 0 || I <= 0 || r < 8 || 2 * r > 128 || r % 8) return 0;
  if (fmt < LORA_W_BF16 || fmt > LORA_W_FP8_E4M3) return 0;
  if (M > (1LL << 31) - 256 || D > (1LL << 30) || I > (1LL << 29)) return 0;
  return mlp_ws_layout(M, D, I, r).total;
}

lora_status_t lora_mlp_fwd(const void* X, int64_t M, const lora_mlp_t* mlp, int32_t r, float s, void* Z, void* GU,
                           void* H, void* XA_gate_up, void* XA_down, void* workspace, size_t ws_bytes, void* stream) {
  TRY(mlp_check(mlp, r, s, M));
  if (M == 0) return LORA_OK;
  TRY(check_ptr(X));
  TRY(check_ptr(Z));
  TRY(check_ptr(GU));
  TRY(check_ptr(H));
  TRY(check_ptr(XA_gate_up));
  TRY(check_ptr(XA_down));
  TRY(mlp_ws_check(M, mlp, r, workspace, ws_bytes));
  const WsLayout wl = mlp_ws_layout(M, mlp->gate_up.K, mlp->down.K, r);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  return mlp_forward_core(X, M, mlp, r, s, Z, GU, H, XA_gate_up, XA_down,
                          reinterpret_cast<__nv_bfloat16*>(ws + wl.skinny_off), reinterpret_cast<float*>(ws + wl.part_off),
                          wl.total - wl.part_off, reinterpret_cast<uint32_t*>(ws), static_cast<cudaStream_t>(stream));
}

static lora_status_t mlp_bwd_entry(const void* dZ, const void* X, void* GU, const void* H, const void* XA_gate_up,
                            const void* XA_down, int64_t M, const lora_mlp_t* mlp, int32_t r, float s, void* dX,
                            void* dA_gate_up, void* dB_gate_up, void* dA_down, void* dB_down, uint32_t flags,
                            void* workspace, size_t ws_bytes, void* stream) {
  if (flags & ~static_cast<uint32_t>(LORA_GRADS_F32)) return LORA_ERR_INVALID_ARG;
  const bool f32 = (flags & LORA_GRADS_F32) != 0;
  TRY(mlp_check(mlp, r, s, M));
  TRY(check_ptr(dA_gate_up));
  TRY(check_ptr(dB_gate_up));
  TRY(check_ptr(dA_down));
  TRY(check_ptr(dB_down));
  const long long D = mlp->gate_up.K, I = mlp->down.K;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (M == 0) {
    const size_t esz = f32 ? 4 : 2;
    const size_t z[4] = {static_cast<size_t>(2 * r) * D * esz, static_cast<size_t>(2 * I) * r * esz,
                         static_cast<size_t>(r) * I * esz, static_cast<size_t>(D) * r * esz};
    void* ptrs[4] = {dA_gate_up, dB_gate_up, dA_down, dB_down};
    for (int i = 0; i < 4; ++i)
      if (cudaMemsetAsync(ptrs[i], 0, z[i], st) != cudaSuccess) return LORA_ERR_CUDA;
    return LORA_OK;
  }
  TRY(check_ptr(dZ));
  TRY(check_ptr(X));
  TRY(check_ptr(GU));
  TRY(check_ptr(H));
  TRY(check_ptr(XA_gate_up));
  TRY(check_ptr(XA_down));
  if (dX) TRY(check_ptr(dX));
  TRY(mlp_ws_check(M, mlp, r, workspace, ws_bytes));
  const WsLayout wl = mlp_ws_layout(M, D, I, r);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  return mlp_backward_core(dZ, X, GU, H, XA_gate_up, XA_down, M, mlp, r, s, dX, dA_gate_up, dB_gate_up, dA_down,
                           dB_down, f32, reinterpret_cast<__nv_bfloat16*>(ws + wl.skinny_off),
                           reinterpret_cast<float*>(ws + wl.part_off), wl.total - wl.part_off,
                           reinterpret_cast<uint32_t*>(ws), st);
}

lora_status_t lora_mlp_bwd(const void* dZ, const void* X, void* GU, const void* H, const void* XA_gate_up,
                           const void* XA_down, int64_t M, const lora_mlp_t* mlp, int32_t r, float s, void* dX,
                           void* dA_gate_up, void* dB_gate_up, void* dA_down, void* dB_down, void* workspace,
                           size_t ws_bytes, void* stream) {
  return mlp_bwd_entry(dZ, X, GU, H, XA_gate_up, XA_down, M, mlp, r, s, dX, dA_gate_up, dB_gate_up, dA_down,
                       dB_down, 0u, workspace, ws_bytes, stream);
}

lora_status_t lora_mlp_bwd_ex(const void* dZ, const void* X, void* GU, const void* H, const void* XA_gate_up,
                              const void* XA_down, int64_t M, const lora_mlp_t* mlp, int32_t r, float s, void* dX,
                              void* dA_gate_up, void* dB_gate_up, void* dA_down, void* dB_down, uint32_t flags,
                              void* workspace, size_t ws_bytes, void* stream) {
  return mlp_bwd_entry(dZ, X, GU, H, XA_gate_up, XA_down, M, mlp, r, s, dX, dA_gate_up, dB_gate_up, dA_down,
                       dB_down, flags, workspace, ws_bytes, stream);
}

size_t lora_ce_workspace_bytes(int64_t M, int64_t D, int64_t V, int64_t chunk) {
  if (M < 0 || D <= 0 || V <= 0 || chunk < 0) return 0;
  if (M > (1LL << 31) - 256 || D > (1LL << 30) || V > (1LL << 31) - 256) return 0;
  const CeLayout c = ce_layout(M, D, V);
  long long vc = chunk == 0 ? V : chunk;
  vc = (vc + 255) / 256 * 256;
  const size_t bwd = c.bwd_fixed + align256(static_cast<size_t>(M) * vc * 2);
  return c.fwd_total > bwd ? c.fwd_total : bwd;
}

lora_status_t lora_ce_fwd(const void* X, int64_t M, const lora_weight_t* W, const int32_t* labels,
                          int32_t ignore_index, float* loss, float* lse, void* workspace, size_t ws_bytes,
                          void* stream) {
  TRY(ce_check(X, M, W, labels));
  if (M == 0) return LORA_OK;
  TRY(check_ptr(loss));
  TRY(check_ptr(lse));
  if (!workspace) return LORA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return LORA_ERR_ALIGNMENT;
  const long long V = W->N, D = W->K;
  const CeLayout c = ce_layout(M, D, V);
  if (ws_bytes < c.fwd_total) return LORA_ERR_WORKSPACE;
  DevInfo* dev = nullptr;
  TRY(dev_info(&dev));
  TRY(get_encode());
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* zy = reinterpret_cast<float*>(ws + c.zy_off);
  // a label outside [0, V) finds no tile: its logit stays NaN and so does its loss
  if (cudaMemsetAsync(zy, 0xFF, static_cast<size_t>(M) * 4, st) != cudaSuccess) return LORA_ERR_CUDA;
  CUtensorMap ta;
  TRY(tmap_bf16(&ta, X, D, M, kBoxX, kBoxY));
  PairParams p = ce_params(M, V, D, nullptr, reinterpret_cast<uint32_t*>(ws), W);
  p.labels = labels;
  p.ignore_index = ignore_index;
  p.lse_part = reinterpret_cast<float*>(ws + c.part_off);
  p.label_logit = zy;
  TRY((launch_gemm_w<false, EPI_CE_LSE>(W, ta, ta, FSpec{X, static_cast<uint64_t>(D), static_cast<uint64_t>(M)}, p,
                                         dev->sms, st)));
  launch_k(ce_finalize_kernel, dim3(cdiv(M, 256)), dim3(256), 0, st, reinterpret_cast<const float2*>(ws + c.part_off),
           cdiv(V, 256), static_cast<int>(M), zy, labels, ignore_index, loss, lse);
  count_launch();
  return last_launch();
}

lora_status_t lora_ce_bwd(const void* X, int64_t M, const lora_weight_t* W, const int32_t* labels,
                          int32_t ignore_index, const float* lse, const float* dloss, void* dX, void* workspace,
                          size_t ws_bytes, void* stream) {
  TRY(ce_check(X, M, W, labels));
  if (M == 0) return LORA_OK;
  TRY(check_ptr(lse));
  TRY(check_ptr(dloss));
  TRY(check_ptr(dX));
  if (!workspace) return LORA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return LORA_ERR_ALIGNMENT;
  const long long V = W->N, D = W->K;
  const CeLayout c = ce_layout(M, D, V);
  // the vocabulary slice: as many 256-column tiles of dlogits as the workspace holds
  if (ws_bytes < c.bwd_fixed) return LORA_ERR_WORKSPACE;
  long long vc = static_cast<long long>((ws_bytes - c.bwd_fixed) / (static_cast<size_t>(M) * 2)) / 256 * 256;
  if (vc < 256) return LORA_ERR_WORKSPACE;
  if (vc > V) vc = V;
  DevInfo* dev = nullptr;
  TRY(dev_info(&dev));
  TRY(get_encode());
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  float* acc = reinterpret_cast<float*>(ws + c.acc_off);
  auto* dlog = reinterpret_cast<__nv_bfloat16*>(ws + c.dlog_off);
  CUtensorMap tx;
  TRY(tmap_bf16(&tx, X, D, M, kBoxX, kBoxY));
  const int nslices = static_cast<int>((V + vc - 1) / vc);
  for (int i = 0; i < nslices; ++i) {
    const long long v0 = i * vc, w = (V - v0 < vc) ? V - v0 : vc;
    lora_weight_t Wc = *W;  // rows [v0, v0 + w) of the head
    Wc.N = w;
    Wc.data = static_cast<const uint8_t*>(W->data) + static_cast<size_t>(v0) * D * 2;
    // dlogits of the slice
    PairParams p = ce_params(M, w, D, dlog, status, &Wc);
    p.labels = labels;
    p.ignore_index = ignore_index;
    p.v0 = static_cast<int>(v0);
    p.lse = lse;
    p.dloss = dloss;
    TRY((launch_gemm_w<false, EPI_CE_DLOGITS>(&Wc, tx, tx, FSpec{X, static_cast<uint64_t>(D), static_cast<uint64_t>(M)},
                                              p, dev->sms, st)));
    // dX (+)= dlogits_slice · W_slice, summed over slices in fp32
    CUtensorMap ta;
    TRY(tmap_bf16(&ta, dlog, w, M, kBoxX, kBoxY));
    PairParams q = ce_params(M, D, w, dX, status, &Wc);
    q.acc32 = acc;
    q.acc_mode = (i > 0 ? 1 : 0) | (i == nslices - 1 ? 2 : 0);
    TRY((launch_gemm_w<true, EPI_ACC_F32>(&Wc, ta, ta, FSpec{dlog, static_cast<uint64_t>(w), static_cast<uint64_t>(M)},
                                          q, dev->sms, st)));
  }
  return LORA_OK;
}

lora_status_t dequant_blockwise4(const lora_weight_t* Wq, void* W_out, void* stream) {
  TRY(check_weight(Wq));
  if (Wq->fmt != LORA_W_BLOCK4) return LORA_ERR_INVALID_ARG;
  TRY(check_ptr(W_out));
  DevInfo* dev = nullptr;
  TRY(dev_info(&dev));
  const size_t total = static_cast<size_t>(Wq->N) * Wq->K;
  const size_t groups = total / 16;
  size_t grid = (groups + 255) / 256;
  const size_t cap = static_cast<size_t>(dev->sms) * 8;
  if (grid > cap) grid = cap;
  dequant4_kernel<<<static_cast<int>(grid), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(Wq->data), static_cast<const __half*>(Wq->absmax), Wq->codebook,
      static_cast<__nv_bfloat16*>(W_out), total);
  count_launch();
  return last_launch();
}

lora_status_t lora_dequant(const lora_weight_t* W, void* W_out, void* stream) {
  TRY(check_weight(W));
  TRY(check_ptr(W_out));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t total = static_cast<size_t>(W->N) * W->K;
  if (W->fmt == LORA_W_BLOCK4) return dequant_blockwise4(W, W_out, stream);
  {
    // the output may not overlap the stored weight
    const uint8_t* c0 = static_cast<const uint8_t*>(W->data);
    const uint8_t* c1 = c0 + total * (W->fmt == LORA_W_BF16 ? 2 : 1);
    const uint8_t* o0 = static_cast<const uint8_t*>(W_out);
    if (o0 < c1 && c0 < o0 + total * 2) return LORA_ERR_INVALID_ARG;
  }
  if (W->fmt == LORA_W_BF16) {
    if (cudaMemcpyAsync(W_out, W->data, total * 2, cudaMemcpyDeviceToDevice, st) != cudaSuccess) return LORA_ERR_CUDA;
    return LORA_OK;
  }
  DevInfo* dev = nullptr;
  TRY(dev_info(&dev));
  const size_t groups = total / 16;
  size_t grid = (groups + 255) / 256;
  const size_t cap = static_cast<size_t>(dev->sms) * 8;
  if (grid > cap) grid = cap;
  const auto* codes = static_cast<const uint8_t*>(W->data);
  const auto* scale = static_cast<const float*>(W->absmax);
  auto* out = static_cast<__nv_bfloat16*>(W_out);
  if (W->fmt == LORA_W_INT8)
    dequant8_kernel<2><<<static_cast<int>(grid), 256, 0, st>>>(codes, scale, out, total, W->K);
  else
    dequant8_kernel<3><<<static_cast<int>(grid), 256, 0, st>>>(codes, scale, out, total, W->K);
  count_launch();
  return last_launch();
}

lora_status_t lora_merge(const lora_weight_t* W, const void* A, const void* B, int32_t r, float s, void* W_out,
                         void* stream) {
  TRY(check_weight(W));
  TRY(check_rank(r, s));
  TRY(check_ptr(A));
  TRY(check_ptr(B));
  TRY(check_ptr(W_out));
  const bool bf = W->fmt == LORA_W_BF16;
  if (!bf) {
    // an output overlapping the codes would be read after it is written
    const uint8_t* c0 = static_cast<const uint8_t*>(W->data);
    const uint8_t* c1 = c0 + static_cast<size_t>(W->N) * W->K / (W->fmt == LORA_W_BLOCK4 ? 2 : 1);
    const uint8_t* o0 = static_cast<const uint8_t*>(W_out);
    const uint8_t* o1 = o0 + static_cast<size_t>(W->N) * W->K * 2;
    if (o0 < c1 && c0 < o1) return LORA_ERR_INVALID_ARG;
  }
  const size_t smem = static_cast<size_t>(MG_TN * r + r * MG_TK) * sizeof(float);
  if (cudaFuncSetAttribute(merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
      cudaSuccess)
    return LORA_ERR_CUDA;
  dim3 grid(cdiv(W->K, MG_TK), cdiv(W->N, MG_TN));
  const bool w4 = W->fmt == LORA_W_BLOCK4;
  merge_kernel<<<grid, MG_THREADS, smem, static_cast<cudaStream_t>(stream)>>>(
      W->fmt, bf ? static_cast<const __nv_bfloat16*>(W->data) : nullptr,
      bf ? nullptr : static_cast<const uint8_t*>(W->data), w4 ? static_cast<const __half*>(W->absmax) : nullptr,
      w4 ? W->codebook : nullptr, (!bf && !w4) ? static_cast<const float*>(W->absmax) : nullptr,
      static_cast<const __nv_bfloat16*>(A), static_cast<const __nv_bfloat16*>(B), static_cast<int>(W->N),
      static_cast<int>(W->K), r, s, static_cast<__nv_bfloat16*>(W_out));
  count_launch();
  return last_launch();
}

lora_status_t lora_device_status(void* workspace, void* stream) {
  if (!workspace) return LORA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return LORA_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess) return LORA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return LORA_ERR_CUDA;
  if (word == 0) return LORA_OK;
  if (cudaMemsetAsync(workspace, 0, sizeof(uint32_t), st) != cudaSuccess) return LORA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return LORA_ERR_CUDA;
  if (word & kDevErrBounds) return LORA_ERR_DEVICE_BOUNDS;
  return (word & kDevErrTimeout) ? LORA_ERR_DEVICE_TIMEOUT : LORA_ERR_CUDA;
}

lora_status_t lora_testing_bounded_wait(void* workspace, uint64_t limit_ns, void* stream) {
  if (!workspace) return LORA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return LORA_ERR_ALIGNMENT;
  if (limit_ns == 0 || limit_ns > 10000000000ull) return LORA_ERR_INVALID_ARG;
  bounded_wait_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<uint32_t*>(workspace), limit_ns);
  count_launch();
  return last_launch();
}

int32_t lora_testing_gemm_streamk(int64_t M, int64_t Nout, int64_t Kred, int32_t r, int32_t fmt) {
  if (fmt < LORA_W_BF16 || fmt > LORA_W_FP8_E4M3 || r < 0 || r > 128) return -1;
  const GemmSched g = gemm_sched(M, Nout, Kred, r, fmt != LORA_W_BF16);
  if (!g.sk) return 0;
  const long long tiles = static_cast<long long>(cdiv(M, g.tile_rows)) * cdiv(Nout, 256);
  return static_cast<int32_t>(tiles - g.dp_tiles);
}

int32_t lora_testing_dual_blocking(int64_t M, int64_t C, int32_t r, int32_t mode, int32_t* out4) {
  if (!out4 || M <= 0 || C <= 0 || r < 1 || r > 128 || mode < DP_BOTH || mode > DP_COLS) return -1;
  const DualSplit d = dual_split(M, C, r, mode);
  out4[0] = d.a;
  out4[1] = d.b;
  out4[2] = d.row_tiles;
  out4[3] = d.col_tiles;
  return d.use ? 1 : 0;
}

lora_status_t lora_testing_tcproj_extra_tile(const void* P, const void* A, int64_t rows, int64_t red, int32_t r,
                                             float* part, size_t part_bytes, void* workspace, void* stream) {
  if (rows <= 0 || red <= 0 || red % 8 != 0 || rows > (1LL << 30) || red > (1LL << 30)) return LORA_ERR_INVALID_ARG;
  if (r <= 16 || r > 128 || r % 8 != 0) return LORA_ERR_UNSUPPORTED;
  TRY(check_ptr(P));
  TRY(check_ptr(A));
  TRY(check_ptr(part));
  if (!workspace) return LORA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return LORA_ERR_ALIGNMENT;
  TcSplit t = tc_split(rows, red, r);
  if (part_bytes < static_cast<size_t>(t.splits) * rows * r * 4) return LORA_ERR_WORKSPACE;
  DevInfo* dev = nullptr;
  TRY(dev_info(&dev));
  TRY(get_encode());
  t.tiles += 1;  // one tile past the last row
  return launch_tcproj<TP_ROWS_K>(static_cast<const __nv_bfloat16*>(P), red, static_cast<const __nv_bfloat16*>(A),
                                  red, rows, red, r, t, part, static_cast<uint32_t*>(workspace),
                                  static_cast<cudaStream_t>(stream));
}

int32_t lora_testing_tcproj_splits(int64_t rows, int64_t red, int32_t r) {
  if (rows <= 0 || red <= 0 || r < 1 || r > 128) return -1;
  return tc_split(rows, red, r).splits;
}

int32_t lora_testing_xpass_tma(int64_t M, int64_t K, int32_t r) {
  if (M <= 0 || K <= 0 || r < 1 || r > 128) return -1;
  return (dual_split(M, K, r, DP_ROWS).use ? 1 : 0) | (dual_split(M, K, r, DP_COLS).use ? 2 : 0);
}

lora_status_t lora_timing_enable(int32_t on) {
  g_timing_on.store(on != 0);
  return LORA_OK;
}

lora_status_t lora_timing_read(int32_t kernel, double* total_ms, int64_t* launches) {
  if (kernel < 0 || kernel >= LORA_KERNEL_COUNT || !total_ms || !launches) return LORA_ERR_INVALID_ARG;
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> ev;
  {
    std::lock_guard<std::mutex> lk(g_timing_mu);
    ev.swap(g_timing[kernel]);
  }
  double tot = 0.0;
  bool ok = true;
  for (auto& pr : ev) {
    float ms = 0.f;
    if (cudaEventSynchronize(pr.second) != cudaSuccess || cudaEventElapsedTime(&ms, pr.first, pr.second) != cudaSuccess)
      ok = false;
    tot += ms;
    cudaEventDestroy(pr.first);
    cudaEventDestroy(pr.second);
  }
  *total_ms = tot;
  *launches = static_cast<int64_t>(ev.size());
  return ok ? LORA_OK : LORA_ERR_CUDA;
}

int64_t lora_launch_count(void) { return g_launches.load(); }

}  // extern "C"

// ---------------------------------------------------------------- forward without allocation
// The fixed scratch of lora_linear_fwd_noalloc.  In host code this name is only a
// stand-in for the symbol; its device address is looked up per device with
// cudaGetSymbolAddress and only that address is handed to kernels.
static __device__ __align__(256) uint8_t g_noalloc_scratch[LORA_NOALLOC_SCRATCH_BYTES];

namespace lora {
namespace {

struct NoAllocLayout {
  size_t sxa_off, part_off, total;
};
NoAllocLayout noalloc_layout(long long M, long long K, int r) {
  NoAllocLayout l;
  l.sxa_off = 0;
  l.part_off = align256(static_cast<size_t>(M) * r * 2);
  l.total = l.part_off + align256(static_cast<size_t>(rowproj_split(M, K).splits) * M * r * 4);
  return l;
}

std::mutex g_noalloc_mu;
void* g_noalloc_addr[64] = {};
CUcontext g_noalloc_ctx[64] = {};

// Device address of the fixed scratch on the current device, looked up on the first
// call in each context (the array lives in the library's module of that context, so a
// context created anew after cudaDeviceReset has its own copy at another address).
lora_status_t noalloc_scratch(uint8_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return LORA_ERR_CUDA;
  const CUcontext ctx = current_ctx();  // current: dev_info() ran first
  if (!ctx) return LORA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_addr[dev] || g_noalloc_ctx[dev] != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return LORA_ERR_CUDA;
    g_noalloc_addr[dev] = p;
    g_noalloc_ctx[dev] = ctx;
  }
  *out = static_cast<uint8_t*>(g_noalloc_addr[dev]);
  return LORA_OK;
}

}  // namespace
}  // namespace lora

extern "C" {

lora_status_t lora_linear_fwd_noalloc(const void* X, int64_t M, const lora_weight_t* W, const void* A, const void* B,
                                      int32_t r, float s, void* Y, void* XA, void* stream) {
  Segs sg;
  TRY(check_common(W, nullptr, r, s, M, A, B, &sg));
  if (M == 0) return LORA_OK;
  TRY(check_ptr(X));
  TRY(check_ptr(Y));
  TRY(check_ptr(XA));
  const NoAllocLayout nl = noalloc_layout(M, W->K, r);
  if (nl.total > LORA_NOALLOC_SCRATCH_BYTES) return LORA_ERR_SCRATCH_LIMIT;
  DevInfo* dev = nullptr;
  TRY(dev_info(&dev));
  uint8_t* scratch = nullptr;
  TRY(noalloc_scratch(&scratch));
  // every scratch byte read below (the split partials, then s·XA) is written earlier in
  // the same call; no status word: an expired device wait ends the kernel silently
  return forward_core(X, M, W, sg, A, B, r, s, Y, XA, reinterpret_cast<__nv_bfloat16*>(scratch + nl.sxa_off),
                      reinterpret_cast<float*>(scratch + nl.part_off), 0, nullptr, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
