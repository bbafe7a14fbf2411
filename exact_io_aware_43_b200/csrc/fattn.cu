// fattn.cu -- host side of libfattn: argument checks, TMA descriptors, launches (C ABI in
// include/fattn.h).  Every step of the attention computation runs in the kernels of fwd.cuh,
// bwd.cuh, bwd_q128.cuh and merge.cuh; this file validates, encodes descriptors, picks the
// schedule (units, key ranges, head groups) and launches, and for fa_fwd_bwd_host orders the
// copies of head chunks around the kernels on its copy streams.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include "../../include/fattn.h"
#include "bwd.cuh"
#include "bwd_q128.cuh"
#include "bwd_pair.cuh"
#include "merge.cuh"
#include "fwd.cuh"
#include "fwd_fp8.cuh"

namespace {

thread_local char g_msg[512] = "";

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(FA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// ---- driver entry point for cuTensorMapEncodeTiled (resolved once through the runtime)
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Tiled map over a contiguous bf16 [BH, N, d] tensor: box = 64 columns (128 bytes, one swizzle
// row) x `box_rows` rows x 1 head, 128-byte swizzle, zero fill past N.
// bf16 [BH, N, d] map, 128-byte swizzle, box 64 columns x box_rows rows x box_heads heads (the
// box's rows land in shared memory head-major: row g * box_rows + i).
int make_map(CUtensorMap* m, const void* base, int BH, int N, int d, int box_rows,
             int box_heads = 1) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(N), cuuint64_t(BH)};
  cuuint64_t strides[2] = {cuuint64_t(d) * 2, cuuint64_t(N) * cuuint64_t(d) * 2};
  cuuint32_t box[3] = {64, cuuint32_t(box_rows), cuuint32_t(box_heads)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return FA_OK;
}

// e4m3 [BH, N, d] map (one byte per element): box = min(d, 128) bytes x box_rows rows x 1 head,
// 128-byte swizzle for d >= 128 (d / 128 boxes across a row), 64-byte swizzle for d = 64.
int make_map_e4m3(CUtensorMap* m, const void* base, int BH, int N, int d, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(N), cuuint64_t(BH)};
  cuuint64_t strides[2] = {cuuint64_t(d), cuuint64_t(N) * cuuint64_t(d)};
  cuuint32_t box[3] = {cuuint32_t(d >= 128 ? 128 : d), cuuint32_t(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  d >= 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled (e4m3) failed (%d)", int(r));
  return FA_OK;
}

// ---- optional per-kernel event timing (benchmark support)
struct KernelTimer {
  std::mutex mu;
  bool on = false;
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> ev[5];
};
KernelTimer g_timer;

struct TimedLaunch {
  int kind;
  cudaStream_t st;
  cudaEvent_t a = nullptr, b = nullptr;
  TimedLaunch(int k, cudaStream_t s) : kind(k), st(s) {
    if (!g_timer.on) return;
    if (cudaEventCreate(&a) != cudaSuccess || cudaEventCreate(&b) != cudaSuccess) {
      a = b = nullptr;
      return;
    }
    cudaEventRecord(a, st);
  }
  ~TimedLaunch() {
    if (!a) return;
    cudaEventRecord(b, st);
    std::lock_guard<std::mutex> g(g_timer.mu);
    g_timer.ev[kind].emplace_back(a, b);
  }
};

// fp32 [BH, N, d] map for the dQ accumulator: box `box_cols` columns x `box_rows` rows x 1 head,
// no swizzle (the reduce-add source in shared memory is a dense [box_rows][box_cols] fp32 tile).
int make_map_f32(CUtensorMap* m, void* base, int BH, int N, int d, int box_cols = 64,
                 int box_rows = 64) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(N), cuuint64_t(BH)};
  cuuint64_t strides[2] = {cuuint64_t(d) * 4, cuuint64_t(N) * cuuint64_t(d) * 4};
  cuuint32_t boxd[3] = {cuuint32_t(box_cols), cuuint32_t(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, boxd, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled (f32) failed (%d)", int(r));
  return FA_OK;
}

// Default bound of every wait inside the kernels: 2 s, far above any legitimate wait.  The test
// build that starves a wait on purpose compiles in a 1 ms default instead.
#ifndef FA_DEFAULT_WAIT_LIMIT_NS
#define FA_DEFAULT_WAIT_LIMIT_NS 2000000000ull
#endif

uint64_t wait_limit_ns() {
  static uint64_t v = [] {
    const char* e = getenv("FA_WAIT_LIMIT_NS");
    uint64_t x = e ? strtoull(e, nullptr, 10) : 0;
    return x ? x : uint64_t(FA_DEFAULT_WAIT_LIMIT_NS);
  }();
  return v;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Grouped heads: H query heads share H_kv key/value heads, H / H_kv consecutive query heads each.
int check_groups(int H, int H_kv) {
  if (H_kv < 1 || H_kv > H || H % H_kv != 0)
    return fail(FA_ERR_INVALID_ARG, "H_kv must divide H (got H=%d, H_kv=%d)", H, H_kv);
  return FA_OK;
}

int check_common(int B, int H, int N, int d, float scale) {
  if (B < 1 || H < 1 || N < 1)
    return fail(FA_ERR_INVALID_ARG, "B, H and N must be >= 1 (got %d, %d, %d)", B, H, N);
  if (d != 64 && d != 128 && d != 256)
    return fail(FA_ERR_UNSUPPORTED, "head dim d=%d is not supported (64, 128 or 256)", d);
  if (!std::isfinite(scale) || !(scale > 0.f))
    return fail(FA_ERR_INVALID_ARG, "scale must be finite and > 0");
  const long long bh = (long long)B * H;
  if (bh > (1ll << 30) || (long long)N > (1ll << 30))
    return fail(FA_ERR_INVALID_ARG, "B*H or N too large");
  const long long blocks = bh * ((N + 127) / 128);
  if (blocks > 0x3fffffffll) return fail(FA_ERR_INVALID_ARG, "problem too large for one grid");
  return FA_OK;
}

int check_device() {
  static thread_local int cached_dev = -1, cached_ok = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev != cached_dev) {
    cudaDeviceProp prop;
    e = cudaGetDeviceProperties(&prop, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceProperties");
    cached_ok = (prop.major == 10 && prop.minor == 0);
    cached_dev = dev;
  }
  if (!cached_ok) return fail(FA_ERR_UNSUPPORTED, "libfattn needs an sm_100 (B200) device");
  return FA_OK;
}

template <typename K>
int set_smem(K kernel, int bytes) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  return FA_OK;
}

#ifndef FA_FWD_PERSISTENT
#define FA_FWD_PERSISTENT 1
#endif

int sm_count() {
  static thread_local int dev_cached = -1, n = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess && dev != dev_cached) {
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    dev_cached = dev;
  }
  return n;
}

// FA_FWD_TAIL_SPLIT: 1 cuts the units of a short last round in two (plain non-causal forward).
#ifndef FA_FWD_TAIL_SPLIT
#define FA_FWD_TAIL_SPLIT 1
#endif

template <int D, bool CAUSAL, int NQT>
int launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
               const CUtensorMap& mo, fattn::FwdParams p, int BH, cudaStream_t st) {
  using C = fattn::FwdCfg<D, NQT>;
  const bool general = p.o_part != nullptr || p.pack > 1;
  auto kern = general ? fattn::fa_fwd_kernel<D, CAUSAL, NQT, true>
                      : fattn::fa_fwd_kernel<D, CAUSAL, NQT, false>;
  int rc = set_smem(kern, C::SMEM_BYTES);
  if (rc) return rc;
  if (C::REALLOC) {
    // setmaxnreg.inc can only draw on the registers the CTA was launched with; refuse to launch
    // a build whose per-thread launch allocation is below the split the kernel asks for.
    // per kernel variant: 0 unknown, 1 ok, 2 bad; threads that race here compute the same value
    static std::atomic<int> checked[2] = {{0}, {0}};
    std::atomic<int>& chk_slot = checked[general ? 1 : 0];
    int chk = chk_slot.load(std::memory_order_relaxed);
    if (chk == 0) {
      cudaFuncAttributes fa_attr;
      cudaError_t e = cudaFuncGetAttributes(&fa_attr, kern);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes");
      chk = (fa_attr.numRegs * C::THREADS >= C::CTRL_REGS * 128 + C::SOFTMAX_REGS * 256) ? 1 : 2;
      chk_slot.store(chk, std::memory_order_relaxed);
    }
    if (chk == 2)
      return fail(FA_ERR_UNSUPPORTED, "fa_fwd kernel built with too few launch registers for its "
                                      "register split");
  }
  p.BH = BH;
  if (p.pack > 1) {
    p.nqb = 1;
    p.units = (BH / p.G) * p.splits;
  } else {
    p.nqb = (p.Nq + NQT * C::BM - 1) / (NQT * C::BM);
    p.units = BH * p.nqb * p.splits;
  }
  p.tail_base = p.units;
  if (FA_FWD_TAIL_SPLIT && !CAUSAL && !general && NQT == 2 && p.units > sm_count()) {
    // the last round of the persistent grid holds `last` units: when that is at most half a
    // round, cut each in two one-tile work items, so the round takes about half as long
    const int g = sm_count();
    const int rounds = (p.units + g - 1) / g;
    const int last = p.units - (rounds - 1) * g;
    if (2 * last <= g) {
      p.tail_base = (rounds - 1) * g;
      p.units = p.tail_base + 2 * last;
    }
  }
  // persistent: one CTA per SM (at most one unit each when there are fewer units than SMs)
  const int G = FA_FWD_PERSISTENT ? (p.units < sm_count() ? p.units : sm_count()) : p.units;
  dim3 grid(static_cast<unsigned>(G));
  TimedLaunch tl(FA_KERNEL_FWD, st);
  kern<<<grid, C::THREADS, C::SMEM_BYTES, st>>>(mq, mk, mv, mo, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "fa_fwd launch");
  return FA_OK;
}

template <int D, bool CAUSAL, int NQT>
int launch_fwd_fp8(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                   fattn::FwdParams p, float v_scale, int BH, cudaStream_t st) {
  using C = fattn::Fp8Cfg<D, NQT>;
  auto kern = fattn::fa_fwd_fp8_kernel<D, CAUSAL, NQT>;
  int rc = set_smem(kern, C::SMEM_BYTES);
  if (rc) return rc;
  if (C::REALLOC) {
    static std::atomic<int> checked{0};  // 0 unknown, 1 ok, 2 bad
    int chk = checked.load(std::memory_order_relaxed);
    if (chk == 0) {
      cudaFuncAttributes fa_attr;
      cudaError_t e = cudaFuncGetAttributes(&fa_attr, kern);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes");
      chk = (fa_attr.numRegs * C::THREADS >= C::CTRL_REGS * 128 + C::SOFTMAX_REGS * 256) ? 1 : 2;
      checked.store(chk, std::memory_order_relaxed);
    }
    if (chk == 2)
      return fail(FA_ERR_UNSUPPORTED, "fa_fwd_fp8 kernel built with too few launch registers for "
                                      "its register split");
  }
  p.BH = BH;
  p.nqb = (p.Nq + NQT * C::BM - 1) / (NQT * C::BM);
  p.units = BH * p.nqb;
  p.tail_base = p.units;  // no split tail: every unit keeps its two query tiles
  const int G = p.units < sm_count() ? p.units : sm_count();
  TimedLaunch tl(FA_KERNEL_FWD, st);
  kern<<<dim3(unsigned(G)), C::THREADS, C::SMEM_BYTES, st>>>(mq, mk, mv, p, v_scale);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "fa_fwd_fp8 launch");
  return FA_OK;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// d = 64 and 128 backward: 128-query steps (fa_bwd_kernel_q128); 0 selects the 64-query kernel.
#ifndef FA_BWD_Q128
#define FA_BWD_Q128 1
#endif
// 128-query backward: 0 launches one CTA per unit (key block, K/V head [, share of a group]);
// 1 launches one CTA per SM that loops over the units; 2 (default) picks the persistent grid
// when units are short (at most kBwdqPersistSteps query-block steps each), where a CTA's set-up,
// K/V load and dK/dV epilogue are a large part of a unit, and one CTA per unit otherwise.
#ifndef FA_BWDQ_PERSIST
#define FA_BWDQ_PERSIST 2
#endif
constexpr int kBwdqPersistSteps = 16;
// K/V heads per band of the unit order on the persistent grid (0: the default band).  Bands of 2
// measured 4x16x2048 causal 663 -> 696 (d = 128), 418 -> 444 (d = 64), GPT-2 shape 283 -> 294.
#ifndef FA_BWDQ_PERSIST_BAND
#define FA_BWDQ_PERSIST_BAND 2
#endif
// d = 256 backward: CTA pairs exchanging P and dS through distributed shared memory
// (fa_bwd_kernel_pair); 0 selects the kernel whose two CTAs per key block each recompute S^T, dP^T.
#ifndef FA_BWD_PAIR
#define FA_BWD_PAIR 1
#endif

template <int D, bool CAUSAL>
int launch_bwd(const void* q, const void* k, const void* v, fattn::BwdParams p, cudaStream_t st) {
  using C = fattn::BwdCfg<D>;
  int rc;
  CUtensorMap mq, mk, mv, mdo;
  if ((rc = make_map(&mq, q, p.BH, p.N, D, C::BR))) return rc;
  if ((rc = make_map(&mk, k, p.BHkv, p.N, D, C::BC))) return rc;
  if ((rc = make_map(&mv, v, p.BHkv, p.N, D, C::BC))) return rc;
  if ((rc = make_map(&mdo, p.dO, p.BH, p.N, D, C::BR))) return rc;
  CUtensorMap mdq;
  if ((rc = make_map_f32(&mdq, p.dq_acc, p.BH, p.N, D))) return rc;
  const int grid_ew = sm_count() * 8;
  {
    TimedLaunch tl(FA_KERNEL_BWD_PRE, st);
    fattn::fa_bwd_pre_kernel<D><<<grid_ew, 256, 0, st>>>(p);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "fa_bwd preprocess launch");
  if ((D == 128 || D == 64) && FA_BWD_Q128) {
    // d = 64, 128: 128-query steps (every GEMM of a step is 128 x 128 x d or 128 x d x 128)
    using CQ = fattn::BwdQ128Cfg<(D == 64 ? 64 : 128)>;
    auto kq = fattn::fa_bwd_kernel_q128<(D == 64 ? 64 : 128), CAUSAL>;
    if ((rc = set_smem(kq, CQ::SMEM_BYTES))) return rc;
    // setmaxnreg.inc draws on the registers the CTA was launched with: refuse a build whose
    // launch allocation is below the kernel's register split
    static std::atomic<int> checked{0};  // 0 unknown, 1 ok, 2 bad
    int chk = checked.load(std::memory_order_relaxed);
    if (chk == 0) {
      cudaFuncAttributes fa_attr;
      e = cudaFuncGetAttributes(&fa_attr, kq);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes");
      chk = (fa_attr.numRegs * CQ::THREADS >=
             CQ::CMP_REGS * 256 + CQ::DQ_REGS * 128 + CQ::CTRL_REGS * 128) ? 1 : 2;
      checked.store(chk, std::memory_order_relaxed);
    }
    if (chk == 2)
      return fail(FA_ERR_UNSUPPORTED, "fa_bwd kernel built with too few launch registers for its "
                                      "register split");
    if ((rc = make_map(&mq, q, p.BH, p.N, D, CQ::BR))) return rc;
    if ((rc = make_map(&mdo, p.dO, p.BH, p.N, D, CQ::BR))) return rc;
    if ((rc = make_map_f32(&mdq, p.dq_acc, p.BH, p.N, D, CQ::DW, 32))) return rc;  // per warp
    // dK, dV written by TMA tensor stores from swizzled shared tiles (same boxes as K, V)
    CUtensorMap mdk, mdv;
    if ((rc = make_map(&mdk, p.dk, p.BHkv, p.N, D, CQ::BC))) return rc;
    if ((rc = make_map(&mdv, p.dv, p.BHkv, p.N, D, CQ::BC))) return rc;
    // one CTA per unit, or (FA_BWDQ_PERSIST) one per SM looping over the units
    const int units = p.BHkv * p.nkb * p.gsplit;
    const int steps_max = p.gq * ((p.N + CQ::BR - 1) / CQ::BR);  // longest unit (non-causal)
    const bool persist =
        FA_BWDQ_PERSIST == 1 || (FA_BWDQ_PERSIST == 2 && steps_max <= kBwdqPersistSteps);
    dim3 grid(unsigned(persist && units > sm_count() ? sm_count() : units));
    fattn::BwdParams pq = p;
    if (persist) pq.head_band = FA_BWDQ_PERSIST_BAND;
    {
      TimedLaunch tl(FA_KERNEL_BWD_MAIN, st);
      kq<<<grid, CQ::THREADS, CQ::SMEM_BYTES, st>>>(mq, mk, mv, mdo, mdq, mdk, mdv, pq);
    }
  } else if (D == 256 && FA_BWD_PAIR) {
    using CP = fattn::BwdPairCfg;
    auto kp = fattn::fa_bwd_kernel_pair<CAUSAL>;
    if ((rc = set_smem(kp, CP::SMEM_BYTES))) return rc;
    if ((rc = make_map(&mq, q, p.BH, p.N, D, CP::BR))) return rc;
    if ((rc = make_map(&mdo, p.dO, p.BH, p.N, D, CP::BR))) return rc;
    if ((rc = make_map(&mk, k, p.BHkv, p.N, D, CP::BC))) return rc;
    if ((rc = make_map(&mv, v, p.BHkv, p.N, D, CP::BC))) return rc;
    if ((rc = make_map_f32(&mdq, p.dq_acc, p.BH, p.N, D, 32, 32))) return rc;  // per drain warp
    CUtensorMap mdk, mdv;  // dK, dV written by TMA tensor stores (same boxes as K, V)
    if ((rc = make_map(&mdk, p.dk, p.BHkv, p.N, D, CP::BC))) return rc;
    if ((rc = make_map(&mdv, p.dv, p.BHkv, p.N, D, CP::BC))) return rc;
    // one cluster of two CTAs per (key block, key/value head [, share of the group's heads])
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2u * unsigned(p.BHkv) * unsigned(p.nkb) * unsigned(p.gsplit));
    cfg.blockDim = dim3(CP::THREADS);
    cfg.dynamicSmemBytes = CP::SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    {
      TimedLaunch tl(FA_KERNEL_BWD_MAIN, st);
      e = cudaLaunchKernelEx(&cfg, kp, mq, mk, mv, mdo, mdq, mdk, mdv, p);
    }
    if (e != cudaSuccess) return cuda_fail(e, "fa_bwd (pair) launch");
  } else {
    auto kern = fattn::fa_bwd_kernel<D, CAUSAL>;
    if ((rc = set_smem(kern, C::SMEM_BYTES))) return rc;
    dim3 grid(unsigned(p.BHkv) * unsigned(p.nkb) * unsigned(C::NSL) * unsigned(p.gsplit));
    {
      TimedLaunch tl(FA_KERNEL_BWD_MAIN, st);
      kern<<<grid, C::THREADS, C::SMEM_BYTES, st>>>(mq, mk, mv, mdo, mdq, p);
    }
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "fa_bwd launch");
  const long long n8 = (long long)p.BH * p.N * D / 8;
  {
    TimedLaunch tl(FA_KERNEL_BWD_POST, st);
    fattn::fa_bwd_post_kernel<<<grid_ew, 256, 0, st>>>(p.dq_acc, p.dq, n8);
    if (p.gsplit > 1) {
      // the group's dK, dV sums were reduced in fp32
      const long long m8 = (long long)p.BHkv * p.N * D / 8;
      fattn::fa_bwd_post_kernel<<<grid_ew, 256, 0, st>>>(p.dk_acc, p.dk, m8);
      fattn::fa_bwd_post_kernel<<<grid_ew, 256, 0, st>>>(p.dv_acc, p.dv, m8);
    }
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "fa_bwd postprocess launch");
  return FA_OK;
}

// KV tiles of 128 keys per split and the number of non-empty splits for a requested count.
int split_chunk(int Nk, int splits) {
  const int tiles = (Nk + 127) / 128;
  const int s = splits < tiles ? splits : tiles;
  return (tiles + s - 1) / s;
}
int effective_splits(int Nk, int splits) {
  if (splits < 1 || Nk < 1) return 0;
  const int tiles = (Nk + 127) / 128;
  const int chunk = split_chunk(Nk, splits);
  return (tiles + chunk - 1) / chunk;
}

// Forward on Nq queries and Nk keys per head (causal: bottom-right aligned, query i sees keys
// j <= i + Nk - Nq) with the keys cut into `splits` ranges; with more than one, partial outputs
// go to o_part / lse_part (see FwdParams) instead of o / lse.
int fwd_launch(const void* q, const void* k, const void* v, void* o, float* lse, float* o_part,
               float* lse_part, int B, int H, int H_kv, int Nq, int Nk, int d, bool causal,
               float scale, int splits, bool pack, cudaStream_t st, bool partials = false) {
  int rc;
  const int BH = B * H;
  const int G = H / H_kv;
  pack = pack && G > 1 && G * Nq <= 128;
  CUtensorMap mq, mk, mv;
  if ((rc = pack ? make_map(&mq, q, BH, Nq, d, Nq, G) : make_map(&mq, q, BH, Nq, d, 128))) return rc;
  if ((rc = make_map(&mk, k, B * H_kv, Nk, d, 128))) return rc;
  if ((rc = make_map(&mv, v, B * H_kv, Nk, d, 128))) return rc;
  // O map for the TMA stores of the plain forward (split and packed outputs store rows
  // directly; they get a placeholder)
  CUtensorMap mo = mq;
  const bool plain_out = !(splits > 1 || partials) && !pack;
  if (plain_out && (rc = make_map(&mo, o, BH, Nq, d, 128))) return rc;
  fattn::FwdParams p{};
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.o_part = (splits > 1 || partials) ? o_part : nullptr;
  p.lse_part = (splits > 1 || partials) ? lse_part : nullptr;
  p.Nq = Nq;
  p.Nk = Nk;
  p.off = Nk - Nq;
  p.H = H;
  p.G = H / H_kv;
  p.splits = splits;
  p.kv_chunk = split_chunk(Nk, splits);
  p.pack = pack ? G : 0;
  p.Hkv = H_kv;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.limit_ns = wait_limit_ns();
  // packed query heads (decoding) fill one query tile only: the one-tile configuration, whose
  // freed second query buffer deepens the K/V ring
  if (d == 64) {
    if (pack)
      return causal ? launch_fwd<64, true, 1>(mq, mk, mv, mo, p, BH, st)
                    : launch_fwd<64, false, 1>(mq, mk, mv, mo, p, BH, st);
    return causal ? launch_fwd<64, true, 2>(mq, mk, mv, mo, p, BH, st)
                  : launch_fwd<64, false, 2>(mq, mk, mv, mo, p, BH, st);
  }
  if (d == 128) {
    if (pack)
      return causal ? launch_fwd<128, true, 1>(mq, mk, mv, mo, p, BH, st)
                    : launch_fwd<128, false, 1>(mq, mk, mv, mo, p, BH, st);
    return causal ? launch_fwd<128, true, 2>(mq, mk, mv, mo, p, BH, st)
                  : launch_fwd<128, false, 2>(mq, mk, mv, mo, p, BH, st);
  }
  return causal ? launch_fwd<256, true, 1>(mq, mk, mv, mo, p, BH, st)
                : launch_fwd<256, false, 1>(mq, mk, mv, mo, p, BH, st);
}

int bwd_dispatch(const void* q, const void* k, const void* v, const void* o, const float* lse,
                 const void* dO, void* dq, void* dk, void* dv, int B, int H, int Hkv, int N, int d,
                 bool causal, float scale, void* workspace, cudaStream_t st) {
  const int BH = B * H;
  fattn::BwdParams p{};
  p.o = static_cast<const __nv_bfloat16*>(o);
  p.dO = static_cast<const __nv_bfloat16*>(dO);
  p.lse = lse;
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  const size_t npad = round_up(size_t(N), 128);
  const size_t dq_bytes = round_up(size_t(BH) * size_t(N) * size_t(d) * 4, 256);
  const size_t row_bytes = round_up(size_t(BH) * npad * 4, 256);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p.dq_acc = reinterpret_cast<float*>(ws);
  p.L2 = reinterpret_cast<float*>(ws + dq_bytes);
  p.Drow = reinterpret_cast<float*>(ws + dq_bytes + row_bytes);
  // d = 64, 128 (128-query kernel): the row statistics as MMA operands, 32 B per padded row
  const size_t aug_bytes = ((d == 128 || d == 64) && FA_BWD_Q128) ? size_t(BH) * npad * 32 : 0;
  p.aug = aug_bytes ? ws + dq_bytes + 2 * row_bytes : nullptr;
  p.BH = BH;
  p.N = N;
  p.Npad = int(npad);
  p.nkb = (N + 127) / 128;
  p.H = H;
  p.Hkv = Hkv;
  p.G = H / Hkv;
  p.BHkv = B * Hkv;
  // grouped heads: when (key blocks x K/V heads) would leave SMs idle, deal each group's query
  // heads out to several CTAs, which reduce their dK, dV sums in fp32 (the workspace of
  // fa_bwd_gqa_workspace_size holds the two accumulators after the row vectors)
  p.gsplit = 1;
  p.gq = p.G;
  static const int gsplit_cap = [] {  // FA_BWD_GSPLIT caps the split (1: off), for comparisons
    const char* e = getenv("FA_BWD_GSPLIT");
    const int x = e ? atoi(e) : 0;
    return x > 0 ? x : 1 << 30;
  }();
  if (p.G > 1 && gsplit_cap > 1) {
    const long long ctas = (long long)p.BHkv * p.nkb * (d == 256 ? 2 : 1);
    const long long target = 2ll * sm_count();
    if (ctas < target) {
      const int want = int((target + ctas - 1) / ctas);
      int gs = want < p.G ? want : p.G;
      if (gs > gsplit_cap) gs = gsplit_cap;
      p.gq = (p.G + gs - 1) / gs;
      p.gsplit = (p.G + p.gq - 1) / p.gq;
    }
  }
  if (p.gsplit > 1) {
    const size_t kv_bytes = round_up(size_t(p.BHkv) * size_t(N) * size_t(d) * 4, 256);
    p.dk_acc = reinterpret_cast<float*>(ws + dq_bytes + 2 * row_bytes + aug_bytes);
    p.dv_acc = reinterpret_cast<float*>(ws + dq_bytes + 2 * row_bytes + aug_bytes + kv_bytes);
  }
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.limit_ns = wait_limit_ns();
  if (d == 64) return causal ? launch_bwd<64, true>(q, k, v, p, st) : launch_bwd<64, false>(q, k, v, p, st);
  if (d == 128)
    return causal ? launch_bwd<128, true>(q, k, v, p, st) : launch_bwd<128, false>(q, k, v, p, st);
  return causal ? launch_bwd<256, true>(q, k, v, p, st) : launch_bwd<256, false>(q, k, v, p, st);
}

}  // namespace

extern "C" {

const char* fa_last_error(void) { return g_msg; }

int fa_version(void) { return 100; }

int fa_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
               int H_kv, int N, int d, int causal, float scale, void* stream) {
  g_msg[0] = 0;
  if (!q || !k || !v || !o || !lse) return fail(FA_ERR_INVALID_ARG, "null tensor pointer");
  int rc = check_common(B, H, N, d, scale);
  if (rc) return rc;
  if ((rc = check_groups(H, H_kv))) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return fail(FA_ERR_MISALIGNED, "tensor pointers must be 16-byte aligned");
  if ((rc = check_device())) return rc;
  return fwd_launch(q, k, v, o, lse, nullptr, nullptr, B, H, H_kv, N, N, d, causal != 0, scale,
                    1, false, static_cast<cudaStream_t>(stream));
}

size_t fa_fwd_splitkv_workspace_size(int B, int H, int Nq, int Nk, int d, int splits) {
  if (B < 1 || H < 1 || Nq < 1 || Nk < 1 || splits < 1 || (d != 64 && d != 128 && d != 256))
    return 0;
  const int eff = effective_splits(Nk, splits);
  if (eff <= 1) return 0;
  const size_t rows = size_t(B) * size_t(H) * size_t(Nq);
  return round_up(size_t(eff) * rows * size_t(d) * 4, 256) + round_up(size_t(eff) * rows * 4, 256);
}

int fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                   int H, int H_kv, int Nq, int Nk, int d, int causal, float scale, int splits,
                   void* workspace, size_t workspace_bytes, void* stream) {
  g_msg[0] = 0;
  if (!q || !k || !v || !o || !lse) return fail(FA_ERR_INVALID_ARG, "null tensor pointer");
  int rc = check_common(B, H, Nq, d, scale);
  if (rc) return rc;
  if ((rc = check_common(B, H, Nk, d, scale))) return rc;
  if ((rc = check_groups(H, H_kv))) return rc;
  if (causal && Nq > Nk)
    return fail(FA_ERR_INVALID_ARG, "causal attention needs Nq <= Nk (got Nq=%d, Nk=%d)", Nq, Nk);
  if (splits < 1) return fail(FA_ERR_INVALID_ARG, "splits must be >= 1 (got %d)", splits);
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return fail(FA_ERR_MISALIGNED, "tensor pointers must be 16-byte aligned");
  const int eff = effective_splits(Nk, splits);
  const size_t need = fa_fwd_splitkv_workspace_size(B, H, Nq, Nk, d, splits);
  if (need && (!workspace || !aligned16(workspace) || workspace_bytes < need))
    return fail(FA_ERR_WORKSPACE, "workspace must be 16-byte aligned and >= %zu bytes", need);
  if ((rc = check_device())) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (eff <= 1)
    return fwd_launch(q, k, v, o, lse, nullptr, nullptr, B, H, H_kv, Nq, Nk, d, causal != 0,
                      scale, 1, true, st);
  const long long rows = (long long)B * H * Nq;
  float* o_part = static_cast<float*>(workspace);
  float* lse_part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                             round_up(size_t(eff) * rows * size_t(d) * 4, 256));
  if ((rc = fwd_launch(q, k, v, o, lse, o_part, lse_part, B, H, H_kv, Nq, Nk, d, causal != 0,
                       scale, eff, true, st)))
    return rc;
  const long long want = (rows + 7) / 8;
  const int blocks = int(want < sm_count() * 16ll ? want : sm_count() * 16ll);
  {
    TimedLaunch tl(FA_KERNEL_FWD_MERGE, st);
    auto* ob = static_cast<__nv_bfloat16*>(o);
    if (d == 64)
      fattn::fa_fwd_merge_kernel<64><<<blocks, 256, 0, st>>>(o_part, lse_part, ob, lse, eff, rows);
    else if (d == 128)
      fattn::fa_fwd_merge_kernel<128><<<blocks, 256, 0, st>>>(o_part, lse_part, ob, lse, eff, rows);
    else
      fattn::fa_fwd_merge_kernel<256><<<blocks, 256, 0, st>>>(o_part, lse_part, ob, lse, eff, rows);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "fa_fwd_splitkv merge launch");
  return FA_OK;
}

int fa_fwd_fp8(const void* q8, const void* k8, const void* v8, float q_scale, float k_scale,
               float v_scale, void* o, float* lse, int B, int H, int N, int d, int causal,
               float scale, void* stream) {
  g_msg[0] = 0;
  if (!q8 || !k8 || !v8 || !o || !lse) return fail(FA_ERR_INVALID_ARG, "null tensor pointer");
  int rc = check_common(B, H, N, d, scale);
  if (rc) return rc;
  for (float x : {q_scale, k_scale, v_scale})
    if (!std::isfinite(x) || !(x > 0.f))
      return fail(FA_ERR_INVALID_ARG, "q_scale, k_scale and v_scale must be finite and > 0");
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v8) || !aligned16(o) || !aligned16(lse))
    return fail(FA_ERR_MISALIGNED, "tensor pointers must be 16-byte aligned");
  if ((rc = check_device())) return rc;
  const int BH = B * H;
  CUtensorMap mq, mk, mv;
  if ((rc = make_map_e4m3(&mq, q8, BH, N, d, 128))) return rc;
  if ((rc = make_map_e4m3(&mk, k8, BH, N, d, 128))) return rc;
  if ((rc = make_map_e4m3(&mv, v8, BH, N, d, 128))) return rc;
  fattn::FwdParams p{};
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.Nq = N;
  p.Nk = N;
  p.off = 0;
  p.H = H;
  p.G = 1;
  p.splits = 1;
  p.kv_chunk = (N + 127) / 128;
  p.Hkv = H;
  p.scale_log2 = scale * q_scale * k_scale * 1.4426950408889634f;
  p.limit_ns = wait_limit_ns();
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d == 64)
    return causal ? launch_fwd_fp8<64, true, 2>(mq, mk, mv, p, v_scale, BH, st)
                  : launch_fwd_fp8<64, false, 2>(mq, mk, mv, p, v_scale, BH, st);
  if (d == 128)
    return causal ? launch_fwd_fp8<128, true, 2>(mq, mk, mv, p, v_scale, BH, st)
                  : launch_fwd_fp8<128, false, 2>(mq, mk, mv, p, v_scale, BH, st);
  return causal ? launch_fwd_fp8<256, true, 1>(mq, mk, mv, p, v_scale, BH, st)
                : launch_fwd_fp8<256, false, 1>(mq, mk, mv, p, v_scale, BH, st);
}

int fa_fwd_partial(const void* q, const void* k, const void* v, float* o_part, float* lse_part,
                   int B, int H, int H_kv, int Nq, int Nk, int d, int causal, float scale,
                   void* stream) {
  g_msg[0] = 0;
  if (!q || !k || !v || !o_part || !lse_part) return fail(FA_ERR_INVALID_ARG, "null tensor pointer");
  int rc = check_common(B, H, Nq, d, scale);
  if (rc) return rc;
  if ((rc = check_common(B, H, Nk, d, scale))) return rc;
  if ((rc = check_groups(H, H_kv))) return rc;
  if (causal && Nq > Nk)
    return fail(FA_ERR_INVALID_ARG, "causal attention needs Nq <= Nk (got Nq=%d, Nk=%d)", Nq, Nk);
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o_part) || !aligned16(lse_part))
    return fail(FA_ERR_MISALIGNED, "tensor pointers must be 16-byte aligned");
  if ((rc = check_device())) return rc;
  return fwd_launch(q, k, v, nullptr, nullptr, o_part, lse_part, B, H, H_kv, Nq, Nk, d,
                    causal != 0, scale, 1, true, static_cast<cudaStream_t>(stream), true);
}

int fa_merge_partials(const float* o_parts, const float* lse_parts, int n_parts, void* o,
                      float* lse, long long rows, int d, void* stream) {
  g_msg[0] = 0;
  if (!o_parts || !lse_parts || !o || !lse) return fail(FA_ERR_INVALID_ARG, "null tensor pointer");
  if (n_parts < 1 || rows < 1)
    return fail(FA_ERR_INVALID_ARG, "n_parts and rows must be >= 1 (got %d, %lld)", n_parts, rows);
  if (d != 64 && d != 128 && d != 256)
    return fail(FA_ERR_UNSUPPORTED, "head dim d=%d is not supported (64, 128 or 256)", d);
  if (!aligned16(o_parts) || !aligned16(lse_parts) || !aligned16(o) || !aligned16(lse))
    return fail(FA_ERR_MISALIGNED, "tensor pointers must be 16-byte aligned");
  int rc = check_device();
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long want = (rows + 7) / 8;
  const int blocks = int(want < sm_count() * 16ll ? want : sm_count() * 16ll);
  {
    TimedLaunch tl(FA_KERNEL_FWD_MERGE, st);
    auto* ob = static_cast<__nv_bfloat16*>(o);
    if (d == 64)
      fattn::fa_fwd_merge_kernel<64><<<blocks, 256, 0, st>>>(o_parts, lse_parts, ob, lse, n_parts, rows);
    else if (d == 128)
      fattn::fa_fwd_merge_kernel<128><<<blocks, 256, 0, st>>>(o_parts, lse_parts, ob, lse, n_parts, rows);
    else
      fattn::fa_fwd_merge_kernel<256><<<blocks, 256, 0, st>>>(o_parts, lse_parts, ob, lse, n_parts, rows);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "fa_merge_partials launch");
  return FA_OK;
}

int fa_selftest_exp2_fma(const float* x, float* y, int n, void* stream) {
  g_msg[0] = 0;
  if (!x || !y || n < 0) return fail(FA_ERR_INVALID_ARG, "null pointer or negative count");
  if (n == 0) return FA_OK;
  int rc = check_device();
  if (rc) return rc;
  const int threads = 256, pairs = (n + 1) / 2;
  fattn::fa_selftest_exp2_fma_kernel<<<(pairs + threads - 1) / threads, threads, 0,
                                       static_cast<cudaStream_t>(stream)>>>(x, y, n);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "fa_selftest_exp2_fma launch");
  return FA_OK;
}

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N,
           int d, int causal, float scale, void* stream) {
  return fa_fwd_gqa(q, k, v, o, lse, B, H, H, N, d, causal, scale, stream);
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1 || (d != 64 && d != 128 && d != 256)) return 0;
  const size_t bh = size_t(B) * size_t(H);
  const size_t npad = round_up(size_t(N), 128);
  const size_t dq = round_up(bh * size_t(N) * size_t(d) * 4, 256);
  const size_t rows = round_up(bh * npad * 4, 256);
  const size_t aug = ((d == 128 || d == 64) && FA_BWD_Q128) ? bh * npad * 32 : 0;
  return dq + 2 * rows + aug;
}

size_t fa_bwd_gqa_workspace_size(int B, int H, int H_kv, int N, int d) {
  const size_t base = fa_bwd_workspace_size(B, H, N, d);
  if (!base || H_kv < 1 || H_kv > H || H % H_kv) return 0;
  if (H_kv == H) return base;
  return base + 2 * round_up(size_t(B) * size_t(H_kv) * size_t(N) * size_t(d) * 4, 256);
}

int fa_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const float* lse,
               const void* dO, void* dq, void* dk, void* dv, int B, int H, int H_kv, int N, int d,
               int causal, float scale, void* workspace, size_t workspace_bytes, void* stream) {
  g_msg[0] = 0;
  if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv)
    return fail(FA_ERR_INVALID_ARG, "null tensor pointer");
  int rc = check_common(B, H, N, d, scale);
  if (rc) return rc;
  if ((rc = check_groups(H, H_kv))) return rc;
  for (const void* ptr : {q, k, v, o, static_cast<const void*>(lse), dO,
                          static_cast<const void*>(dq), static_cast<const void*>(dk),
                          static_cast<const void*>(dv)})
    if (!aligned16(ptr)) return fail(FA_ERR_MISALIGNED, "tensor pointers must be 16-byte aligned");
  const size_t need = fa_bwd_gqa_workspace_size(B, H, H_kv, N, d);
  if (!workspace || !aligned16(workspace) || workspace_bytes < need)
    return fail(FA_ERR_WORKSPACE, "workspace must be 16-byte aligned and >= %zu bytes", need);
  if ((rc = check_device())) return rc;
  return bwd_dispatch(q, k, v, o, lse, dO, dq, dk, dv, B, H, H_kv, N, d, causal != 0, scale,
                      workspace, static_cast<cudaStream_t>(stream));
}

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
           const void* dO, void* dq, void* dk, void* dv, int B, int H, int N, int d, int causal,
           float scale, void* workspace, size_t workspace_bytes, void* stream) {
  return fa_bwd_gqa(q, k, v, o, lse, dO, dq, dk, dv, B, H, H, N, d, causal, scale, workspace,
                    workspace_bytes, stream);
}

int fa_timer_enable(int on) {
  std::lock_guard<std::mutex> g(g_timer.mu);
  g_timer.on = on != 0;
  return FA_OK;
}

int fa_timer_read(int kernel, int* launches, double* total_ms) {
  if (kernel < 0 || kernel > 4 || !launches || !total_ms)
    return fail(FA_ERR_INVALID_ARG, "fa_timer_read: bad kernel kind or null output");
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> evs;
  {
    std::lock_guard<std::mutex> g(g_timer.mu);
    evs.swap(g_timer.ev[kernel]);
  }
  double sum = 0.0;
  int rc = FA_OK;
  for (auto& pr : evs) {
    float ms = 0.f;
    cudaError_t e = cudaEventSynchronize(pr.second);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, pr.first, pr.second);
    if (e != cudaSuccess && rc == FA_OK) rc = cuda_fail(e, "fa_timer_read");
    sum += ms;
    cudaEventDestroy(pr.first);
    cudaEventDestroy(pr.second);
  }
  *launches = int(evs.size());
  *total_ms = sum;
  return rc;
}

int fa_device_status(void* stream) {
  g_msg[0] = 0;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int h[2] = {0, 0};
  e = cudaMemcpyFromSymbol(h, fattn::g_status, sizeof(h));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyFromSymbol");
  if (h[0] != 0) {
    int z[2] = {0, 0};
    cudaMemcpyToSymbol(fattn::g_status, z, sizeof(z));
    return fail(h[0], "a kernel abandoned a bounded wait (site %d)", h[1]);
  }
  return FA_OK;
}

}  // extern "C"

// ------------------------------------------------------------------------------------------
// fa_bwd_noalloc: fa_bwd with its workspace in a static device array (callers that cannot
// allocate).  Host code never uses the array's name as an address: the device address comes
// from cudaGetSymbolAddress, looked up once per device with that device current.
// ------------------------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

namespace {

int noalloc_scratch(void** out) {
  static std::mutex mu;
  static void* ptrs[128] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 128) return fail(FA_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> g(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(scratch)");
    ptrs[dev] = p;
  }
  *out = ptrs[dev];
  return FA_OK;
}

}  // namespace

extern "C" int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                              const float* lse, const void* dO, void* dq, void* dk, void* dv,
                              int B, int H, int N, int d, int causal, float scale, void* stream) {
  g_msg[0] = 0;
  if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv)
    return fail(FA_ERR_INVALID_ARG, "null tensor pointer");
  int rc = check_common(B, H, N, d, scale);
  if (rc) return rc;
  for (const void* ptr : {q, k, v, o, static_cast<const void*>(lse), dO,
                          static_cast<const void*>(dq), static_cast<const void*>(dk),
                          static_cast<const void*>(dv)})
    if (!aligned16(ptr)) return fail(FA_ERR_MISALIGNED, "tensor pointers must be 16-byte aligned");
  const size_t need = fa_bwd_workspace_size(B, H, N, d);
  if (need > FA_NOALLOC_SCRATCH_BYTES)
    return fail(FA_ERR_WORKSPACE,
                "fa_bwd_noalloc: this shape needs %zu bytes of scratch but the library's static "
                "scratch holds %u bytes; use fa_bwd with a caller-provided workspace",
                need, unsigned(FA_NOALLOC_SCRATCH_BYTES));
  if ((rc = check_device())) return rc;
  void* ws = nullptr;
  if ((rc = noalloc_scratch(&ws))) return rc;
  return bwd_dispatch(q, k, v, o, lse, dO, dq, dk, dv, B, H, H, N, d, causal != 0, scale, ws,
                      static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------------------------------------
// fa_fwd_bwd_host: forward + backward from host buffers, copies overlapped with the kernels.
// Heads are independent, so the B*H heads are cut into chunks of consecutive heads: chunk c's
// inputs go up on one copy stream while chunk c-1 runs on the caller's stream and chunk c-2's
// gradients come down on another copy stream (host->device and device->host use separate copy
// engines).  Streams and events are host-side objects created once per device and reused.
// ------------------------------------------------------------------------------------------
namespace {

struct HostPipe {
  cudaStream_t in = nullptr, out = nullptr;
  std::vector<cudaEvent_t> ev;  // 3 per chunk + 1
};

int host_pipe(int dev, int nev, HostPipe** out) {
  static std::mutex mu;
  static HostPipe pipes[128];
  if (dev < 0 || dev >= 128) return fail(FA_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> g(mu);
  HostPipe& hp = pipes[dev];
  cudaError_t e;
  if (!hp.in) {
    if ((e = cudaStreamCreateWithFlags(&hp.in, cudaStreamNonBlocking)) != cudaSuccess)
      return cuda_fail(e, "cudaStreamCreateWithFlags");
    if ((e = cudaStreamCreateWithFlags(&hp.out, cudaStreamNonBlocking)) != cudaSuccess)
      return cuda_fail(e, "cudaStreamCreateWithFlags");
  }
  while (int(hp.ev.size()) < nev) {
    cudaEvent_t x;
    if ((e = cudaEventCreateWithFlags(&x, cudaEventDisableTiming)) != cudaSuccess)
      return cuda_fail(e, "cudaEventCreateWithFlags");
    hp.ev.push_back(x);
  }
  *out = &hp;
  return FA_OK;
}

struct HostLayout {
  size_t q, k, v, dO, o, lse, dq, dk, dv, ws, total;
};

HostLayout host_layout(int B, int H, int N, int d, int chunks) {
  HostLayout L{};
  const size_t bh = size_t(B) * size_t(H);
  const size_t t = round_up(bh * size_t(N) * size_t(d) * 2, 256);
  const int hc = int((bh + size_t(chunks) - 1) / size_t(chunks));
  size_t off = 0;
  for (size_t* f : {&L.q, &L.k, &L.v, &L.dO, &L.o, &L.dq, &L.dk, &L.dv}) {
    *f = off;
    off += t;
  }
  L.lse = off;
  off += round_up(bh * size_t(N) * 4, 256);
  L.ws = off;
  off += round_up(fa_bwd_workspace_size(1, hc, N, d), 256);
  L.total = off;
  return L;
}

}  // namespace

extern "C" size_t fa_fwd_bwd_host_device_bytes(int B, int H, int N, int d, int chunks) {
  if (B < 1 || H < 1 || N < 1 || chunks < 1 || (long long)chunks > (long long)B * H ||
      (d != 64 && d != 128 && d != 256))
    return 0;
  return host_layout(B, H, N, d, chunks).total;
}

extern "C" int fa_fwd_bwd_host(const void* q, const void* k, const void* v, const void* dO,
                               void* o, float* lse, void* dq, void* dk, void* dv, int B, int H,
                               int N, int d, int causal, float scale, int chunks,
                               void* device_buffer, size_t device_bytes, void* stream) {
  g_msg[0] = 0;
  if (!q || !k || !v || !dO || !dq || !dk || !dv)
    return fail(FA_ERR_INVALID_ARG, "null tensor pointer");
  int rc = check_common(B, H, N, d, scale);
  if (rc) return rc;
  if (chunks < 1 || (long long)chunks > (long long)B * H)
    return fail(FA_ERR_INVALID_ARG, "chunks must be in [1, B*H] (got %d)", chunks);
  const HostLayout L = host_layout(B, H, N, d, chunks);
  if (!device_buffer || (reinterpret_cast<uintptr_t>(device_buffer) & 255u) ||
      device_bytes < L.total)
    return fail(FA_ERR_WORKSPACE, "device buffer must be 256-byte aligned and >= %zu bytes",
                L.total);
  if ((rc = check_device())) return rc;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  HostPipe* hp = nullptr;
  if ((rc = host_pipe(dev, 3 * chunks + 1, &hp))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(device_buffer);
  const long long bh = (long long)B * H;
  const size_t head_elems = size_t(N) * size_t(d);
  const size_t ws_bytes = round_up(fa_bwd_workspace_size(1, int((bh + chunks - 1) / chunks), N, d), 256);
  // everything starts after the work already queued on the caller's stream
  if ((e = cudaEventRecord(hp->ev[0], st)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  if ((e = cudaStreamWaitEvent(hp->in, hp->ev[0], 0)) != cudaSuccess)
    return cuda_fail(e, "cudaStreamWaitEvent");
  for (int c = 0; c < chunks; ++c) {
    const long long h0 = bh * c / chunks, h1 = bh * (c + 1) / chunks;
    const int hc = int(h1 - h0);
    const size_t eoff = size_t(h0) * head_elems * 2;  // byte offset of the chunk's first head
    const size_t ebytes = size_t(hc) * head_elems * 2;
    cudaEvent_t ev_in = hp->ev[1 + 3 * c], ev_comp = hp->ev[2 + 3 * c], ev_out = hp->ev[3 + 3 * c];
    const void* src[4] = {q, k, v, dO};
    const size_t dst_off[4] = {L.q, L.k, L.v, L.dO};
    for (int t = 0; t < 4; ++t)
      if ((e = cudaMemcpyAsync(base + dst_off[t] + eoff, static_cast<const uint8_t*>(src[t]) + eoff,
                               ebytes, cudaMemcpyHostToDevice, hp->in)) != cudaSuccess)
        return cuda_fail(e, "cudaMemcpyAsync (to device)");
    if ((e = cudaEventRecord(ev_in, hp->in)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    if ((e = cudaStreamWaitEvent(st, ev_in, 0)) != cudaSuccess)
      return cuda_fail(e, "cudaStreamWaitEvent");
    uint8_t* q_dev = base + L.q + eoff;
    float* lse_c = reinterpret_cast<float*>(base + L.lse) + size_t(h0) * N;
    if ((rc = fa_fwd(q_dev, base + L.k + eoff, base + L.v + eoff, base + L.o + eoff, lse_c, 1, hc,
                     N, d, causal, scale, st)))
      return rc;
    if ((rc = fa_bwd(q_dev, base + L.k + eoff, base + L.v + eoff, base + L.o + eoff, lse_c,
                     base + L.dO + eoff, base + L.dq + eoff, base + L.dk + eoff,
                     base + L.dv + eoff, 1, hc, N, d, causal, scale, base + L.ws, ws_bytes, st)))
      return rc;
    if ((e = cudaEventRecord(ev_comp, st)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    if ((e = cudaStreamWaitEvent(hp->out, ev_comp, 0)) != cudaSuccess)
      return cuda_fail(e, "cudaStreamWaitEvent");
    void* dsts[5] = {dq, dk, dv, o, nullptr};
    const size_t srco[4] = {L.dq, L.dk, L.dv, L.o};
    for (int t = 0; t < 4; ++t) {
      if (!dsts[t]) continue;  // o is optional
      if ((e = cudaMemcpyAsync(static_cast<uint8_t*>(dsts[t]) + eoff, base + srco[t] + eoff, ebytes,
                               cudaMemcpyDeviceToHost, hp->out)) != cudaSuccess)
        return cuda_fail(e, "cudaMemcpyAsync (to host)");
    }
    if (lse && (e = cudaMemcpyAsync(lse + size_t(h0) * N, lse_c, size_t(hc) * N * 4,
                                    cudaMemcpyDeviceToHost, hp->out)) != cudaSuccess)
      return cuda_fail(e, "cudaMemcpyAsync (to host)");
    if ((e = cudaEventRecord(ev_out, hp->out)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  }
  // the caller's stream completes after the last copy to the host
  if ((e = cudaStreamWaitEvent(st, hp->ev[3 * chunks], 0)) != cudaSuccess)
    return cuda_fail(e, "cudaStreamWaitEvent");
  return FA_OK;
}

#ifdef FA_TRACE
// Trace build only: copy out (all per-warp slots) and clear the pipeline trace.
extern "C" int fa_trace_read(unsigned long long* host, int max_records) {
  cudaDeviceSynchronize();
  int n = (int)fattn::kTraceMax;
  if (n > max_records) n = max_records;
  cudaMemcpyFromSymbol(host, fattn::g_trace, sizeof(unsigned long long) * 2 * n);
  static unsigned long long zeros[2 * fattn::kTraceMax];
  cudaMemcpyToSymbol(fattn::g_trace, zeros, sizeof(zeros));
  return n;
}
#endif
