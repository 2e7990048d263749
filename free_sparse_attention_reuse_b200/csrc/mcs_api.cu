// C ABI of the MC-Sparse library: argument checks, workspace layout and launch order.
// The declarations and their documentation are in include/mcs.h.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/mcs.h"
#include "attn.cuh"
#include "kmeans.cuh"
#include "pddp.cuh"
#include "select.cuh"

namespace {

using namespace mcs;

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool probed = false;
  bool supported = false;
  int sms = 0;
  bool attrs_set = false;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;

mcs_status current_device(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MCS_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& di = g_dev[dev];
  if (!di.probed) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return MCS_ERR_CUDA;
    di.probed = true;
    di.supported = (major == 10 && minor == 0);
    di.sms = sms;
  }
  if (!di.supported) return MCS_ERR_UNSUPPORTED_ARCH;
  if (!di.attrs_set) {
    bool ok = true;
    ok &= cudaFuncSetAttribute(attn_kernel<64, kDense>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               AttnSmem<64>::BYTES) == cudaSuccess;
    ok &= cudaFuncSetAttribute(attn_kernel<64, kReuse>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               AttnSmem<64>::BYTES) == cudaSuccess;
    ok &= cudaFuncSetAttribute(attn_kernel<64, kResidual>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               AttnSmem<64>::BYTES) == cudaSuccess;
    ok &= cudaFuncSetAttribute(attn_kernel<128, kDense>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               AttnSmem<128>::BYTES) == cudaSuccess;
    ok &= cudaFuncSetAttribute(attn_kernel<128, kReuse>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               AttnSmem<128>::BYTES) == cudaSuccess;
    ok &= cudaFuncSetAttribute(attn_kernel<128, kResidual>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               AttnSmem<128>::BYTES) == cudaSuccess;
    ok &= cudaFuncSetAttribute(select_kernel<64, 64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               SelectSmem<64>::BYTES) == cudaSuccess;
    ok &= cudaFuncSetAttribute(select_kernel<64, 128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               SelectSmem<64>::BYTES) == cudaSuccess;
    ok &= cudaFuncSetAttribute(select_kernel<128, 64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               SelectSmem<128>::BYTES) == cudaSuccess;
    ok &= cudaFuncSetAttribute(select_kernel<128, 128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               SelectSmem<128>::BYTES) == cudaSuccess;
    ok &= cudaFuncSetAttribute(select_kernel<64, 64, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               SelectSmem<64>::BYTES) == cudaSuccess;
    ok &= cudaFuncSetAttribute(select_kernel<64, 128, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               SelectSmem<64>::BYTES) == cudaSuccess;
    ok &= cudaFuncSetAttribute(select_kernel<128, 64, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               SelectSmem<128>::BYTES) == cudaSuccess;
    ok &= cudaFuncSetAttribute(select_kernel<128, 128, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               SelectSmem<128>::BYTES) == cudaSuccess;
    ok &= cudaFuncSetAttribute(pddp_gram_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(PddpGramSmem<64>::BYTES)) == cudaSuccess;
    ok &= cudaFuncSetAttribute(pddp_gram_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(PddpGramSmem<128>::BYTES)) == cudaSuccess;
    ok &= cudaFuncSetAttribute(pddp_power_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(PddpPowerSmem<64>::BYTES)) == cudaSuccess;
    ok &= cudaFuncSetAttribute(pddp_power_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(PddpPowerSmem<128>::BYTES)) == cudaSuccess;
    // The attention kernels move registers between their warpgroups with setmaxnreg, which
    // draws on the registers the CTA was launched with: the split is sized for 128 per thread
    // (512 x 128 = 65536).  A build whose kernel got another count would make the softmax
    // warpgroups wait for registers that never come, so such a build is refused here.
    auto regs_ok = [](const void* fn) {
      cudaFuncAttributes fa{};
      return cudaFuncGetAttributes(&fa, fn) == cudaSuccess &&
             static_cast<long long>(fa.numRegs) * kAttnThreads == 65536;
    };
    ok &= regs_ok(reinterpret_cast<const void*>(attn_kernel<64, kDense>));
    ok &= regs_ok(reinterpret_cast<const void*>(attn_kernel<64, kReuse>));
    ok &= regs_ok(reinterpret_cast<const void*>(attn_kernel<64, kResidual>));
    ok &= regs_ok(reinterpret_cast<const void*>(attn_kernel<128, kDense>));
    ok &= regs_ok(reinterpret_cast<const void*>(attn_kernel<128, kReuse>));
    ok &= regs_ok(reinterpret_cast<const void*>(attn_kernel<128, kResidual>));
    auto sel_regs_ok = [](const void* fn) {
      cudaFuncAttributes fa{};
      return cudaFuncGetAttributes(&fa, fn) == cudaSuccess &&
             static_cast<uint32_t>(fa.numRegs) == kSelLaunchRegs;
    };
    ok &= sel_regs_ok(reinterpret_cast<const void*>(select_kernel<64, 64>));
    ok &= sel_regs_ok(reinterpret_cast<const void*>(select_kernel<64, 128>));
    ok &= sel_regs_ok(reinterpret_cast<const void*>(select_kernel<128, 64>));
    ok &= sel_regs_ok(reinterpret_cast<const void*>(select_kernel<128, 128>));
    ok &= sel_regs_ok(reinterpret_cast<const void*>(select_kernel<64, 64, true>));
    ok &= sel_regs_ok(reinterpret_cast<const void*>(select_kernel<64, 128, true>));
    ok &= sel_regs_ok(reinterpret_cast<const void*>(select_kernel<128, 64, true>));
    ok &= sel_regs_ok(reinterpret_cast<const void*>(select_kernel<128, 128, true>));
    ok &= cudaFuncSetAttribute(kmeans_dist_kernel<64, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(KmeansSmem<64>::BYTES)) == cudaSuccess;
    ok &= cudaFuncSetAttribute(kmeans_dist_kernel<64, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(KmeansSmem<64>::BYTES)) == cudaSuccess;
    ok &= cudaFuncSetAttribute(kmeans_dist_kernel<128, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(KmeansSmem<128>::BYTES)) == cudaSuccess;
    ok &= cudaFuncSetAttribute(kmeans_dist_kernel<128, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(KmeansSmem<128>::BYTES)) == cudaSuccess;
    if (!ok) return MCS_ERR_CUDA;
    di.attrs_set = true;
  }
  *out = &di;
  return MCS_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Bound on any single wait of the attention kernels launched from now on, and the flag they
// wait for first (mcs_set_attn_wait_limit).
std::atomic<unsigned long long> g_attn_wait_ns{kWaitLimitNs};
std::atomic<const uint32_t*> g_attn_hold{nullptr};

// cuTensorMapEncodeTiled, reached through the runtime's driver entry point (no libcuda link).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// [rows, d] bf16 view of a [B, H, N, d] tensor, 64-column boxes of `box_rows` rows, 128-byte
// swizzle (the layout the UMMA descriptors expect), zero fill out of bounds.
bool make_row_map(CUtensorMap* m, const void* base, uint64_t rows, int d, uint32_t box_rows,
                  CUtensorMapL2promotion promo = CU_TENSOR_MAP_L2_PROMOTION_L2_256B) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), rows};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, promo,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline float resolve_scale(const mcs_shape& s) {
  return s.scale > 0.f ? s.scale : 1.0f / std::sqrt(static_cast<float>(s.d));
}
constexpr float kLog2e = 1.4426950408889634f;

mcs_status check_shape(const mcs_shape& s) {
  if (s.B < 1 || s.H < 1 || s.N < 1) return MCS_ERR_INVALID_ARG;
  if (s.d != 64 && s.d != 128) return MCS_ERR_SHAPE;
  if (static_cast<long long>(s.B) * s.H > 65535) return MCS_ERR_SHAPE;
  // 32-bit element offsets inside a head (key * d) and TMA row extents (B*H*N) stay in range
  if (s.N > (1 << 24) || static_cast<long long>(s.B) * s.H * s.N > 0xFFFFFFFFll) return MCS_ERR_SHAPE;
  return MCS_OK;
}
mcs_status check_groups(const mcs_shape& s, int C) {
  if (C != 64 && C != 128) return MCS_ERR_SHAPE;
  if (s.N % C != 0) return MCS_ERR_SHAPE;
  return MCS_OK;
}
mcs_status check_k(const mcs_shape& s, int k) { return (k < 1 || k > s.N) ? MCS_ERR_INVALID_ARG : MCS_OK; }

int pddp_levels(int G) {
  int L = 0;
  while ((1 << L) < G) ++L;
  return L;
}

// Workspace carve-up (every part 256-byte aligned).
struct Workspace {
  size_t lse = 0, tmp = 0, keys = 0, psum = 0, pgram = 0, nsum = 0, ngram = 0, mu = 0, vdir = 0, scores = 0,
         total = 0;
  int gram_elems = 0, sel_grid = 0;
  size_t score_stride = 0;
};

Workspace layout(const mcs_shape& s, int C, int sms) {
  Workspace w;
  const size_t BH = static_cast<size_t>(s.B) * s.H, N = s.N, d = s.d;
  const int G = s.N / C;
  w.gram_elems = s.d * (s.d + 1) / 2;
  w.sel_grid = static_cast<int>(std::min<size_t>(BH * G, static_cast<size_t>(sms)));
  w.score_stride = round_up(N, 64);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = round_up(off + bytes, 256);
    return o;
  };
  w.lse = take(BH * N * 4);
  w.tmp = take(BH * N * 4);
  w.keys = take(BH * N * 8);
  w.psum = take(BH * G * d * 8);  // column sums of each chunk, by chunk-leader group
  w.pgram = take(BH * G * static_cast<size_t>(w.gram_elems) * 8);  // one slot per chunk-leader group
  w.nsum = take(BH * G * d * 8);                                    // node totals kept for the next depth
  w.ngram = take(BH * G * static_cast<size_t>(w.gram_elems) * 8);
  w.mu = take(BH * G * d * 8);
  w.vdir = take(BH * G * d * 8);
  w.scores = take(static_cast<size_t>(w.sel_grid) * 2 * w.score_stride * 4);
  w.total = off;
  return w;
}

mcs_status launch_status() { return cudaGetLastError() == cudaSuccess ? MCS_OK : MCS_ERR_CUDA; }

template <int HD, int MODE>
mcs_status run_attn(const AttnParams& p, cudaStream_t st, int sms) {
  const int grid = std::min(p.num_units, sms);
  alignas(64) CUtensorMap tmK, tmV;
  const uint64_t rows = static_cast<uint64_t>(p.BH) * p.N;
  const uint32_t box_rows = kTile;  // whole 128-row tiles (the dense mode's TMA loads)
  if (!make_row_map(&tmK, p.K, rows, HD, box_rows) || !make_row_map(&tmV, p.V, rows, HD, box_rows))
    return MCS_ERR_CUDA;
  attn_kernel<HD, MODE><<<grid, kAttnThreads, AttnSmem<HD>::BYTES, st>>>(tmK, tmV, p);
  return launch_status();
}

template <int MODE>
mcs_status dispatch_attn(int d, const AttnParams& p, cudaStream_t st, int sms) {
  return d == 64 ? run_attn<64, MODE>(p, st, sms) : run_attn<128, MODE>(p, st, sms);
}

mcs_status dense_impl(const mcs_shape& s, const void* Q, const void* K, const void* V, void* O, float* lse,
                      cudaStream_t st, int sms) {
  AttnParams p{};
  p.Q = static_cast<const __nv_bfloat16*>(Q);
  p.K = static_cast<const __nv_bfloat16*>(K);
  p.V = static_cast<const __nv_bfloat16*>(V);
  p.out = static_cast<__nv_bfloat16*>(O);
  p.lse = lse;
  p.BH = s.B * s.H;
  p.N = s.N;
  p.C = kTile;
  p.units_per_head = (s.N + kTile - 1) / kTile;
  p.kv_tiles = p.units_per_head;
  p.kv_count = s.N;
  p.num_units = p.BH * p.units_per_head;
  p.scale_log2 = resolve_scale(s) * kLog2e;
  p.wait_ns = g_attn_wait_ns.load();
  p.hold = g_attn_hold.load();
  p.store_out = O != nullptr;
  return dispatch_attn<kDense>(s.d, p, st, sms);
}

mcs_status sparse_impl(const mcs_shape& s, const void* Q, const void* K, const void* V, const int32_t* perm,
                       int C, const int32_t* idx, int k, const void* R_in, const void* O_full, void* out,
                       bool residual, cudaStream_t st, int sms) {
  AttnParams p{};
  p.Q = static_cast<const __nv_bfloat16*>(Q);
  p.K = static_cast<const __nv_bfloat16*>(K);
  p.V = static_cast<const __nv_bfloat16*>(V);
  p.perm = perm;
  p.idx = idx;
  p.R_in = static_cast<const __nv_bfloat16*>(R_in);
  p.O_full = static_cast<const __nv_bfloat16*>(O_full);
  p.out = static_cast<__nv_bfloat16*>(out);
  p.BH = s.B * s.H;
  p.N = s.N;
  p.C = C;
  p.G = s.N / C;
  p.k = k;
  p.units_per_head = p.G;
  p.kv_tiles = (k + kTile - 1) / kTile;
  p.kv_count = k;
  p.num_units = p.BH * p.G;
  p.scale_log2 = resolve_scale(s) * kLog2e;
  p.wait_ns = g_attn_wait_ns.load();
  p.hold = g_attn_hold.load();
  p.store_out = 1;
  return residual ? dispatch_attn<kResidual>(s.d, p, st, sms) : dispatch_attn<kReuse>(s.d, p, st, sms);
}

template <int D>
mcs_status group_levels(const PddpParams& base, int32_t* perm, int32_t* tmp, cudaStream_t st) {
  const int L = pddp_levels(base.G);
  const long long total = static_cast<long long>(base.BH) * base.N;
  const int init_grid = static_cast<int>(std::min<long long>((total + 255) / 256, 4096));
  if (L == 0) {
    pddp_init_kernel<<<init_grid, 256, 0, st>>>(perm, base.N, total);
    return launch_status();
  }
  int32_t* dst0 = ((L - 1) % 2 == 0) ? perm : tmp;
  int32_t* src = dst0 == perm ? tmp : perm;
  pddp_init_kernel<<<init_grid, 256, 0, st>>>(src, base.N, total);
  if (launch_status() != MCS_OK) return MCS_ERR_CUDA;
  const dim3 grid(base.G, base.BH);
  for (int l = 0; l < L; ++l) {
    PddpParams p = base;
    p.level = l;
    int32_t* dst = ((L - 1 - l) % 2 == 0) ? perm : tmp;
    p.cur = src;
    p.nxt = dst;
    pddp_gram_kernel<D><<<grid, 256, PddpGramSmem<D>::BYTES, st>>>(p);
    pddp_power_kernel<D><<<grid, 256, PddpPowerSmem<D>::BYTES, st>>>(p);
    pddp_project_kernel<D><<<grid, std::max(p.C, D), 0, st>>>(p);
    pddp_split_kernel<D><<<grid, 512, 0, st>>>(p);
    if (launch_status() != MCS_OK) return MCS_ERR_CUDA;
    src = dst;
  }
  return MCS_OK;
}

mcs_status group_impl(const mcs_shape& s, const void* Q, int C, int32_t* perm, char* ws, const Workspace& w,
                      cudaStream_t st) {
  PddpParams p{};
  p.Q = static_cast<const __nv_bfloat16*>(Q);
  p.psum = reinterpret_cast<double*>(ws + w.psum);
  p.pgram = reinterpret_cast<double*>(ws + w.pgram);
  p.nsum = reinterpret_cast<double*>(ws + w.nsum);
  p.ngram = reinterpret_cast<double*>(ws + w.ngram);
  p.mu = reinterpret_cast<double*>(ws + w.mu);
  p.vdir = reinterpret_cast<double*>(ws + w.vdir);
  p.keys = reinterpret_cast<unsigned long long*>(ws + w.keys);
  p.BH = s.B * s.H;
  p.N = s.N;
  p.C = C;
  p.G = s.N / C;
  p.d = s.d;
  p.gram_elems = w.gram_elems;
  int32_t* tmp = reinterpret_cast<int32_t*>(ws + w.tmp);
  return s.d == 64 ? group_levels<64>(p, perm, tmp, st) : group_levels<128>(p, perm, tmp, st);
}

mcs_status select_impl(const mcs_shape& s, const void* Q, const void* K, const int32_t* perm, int C, int k,
                       const float* lse, int32_t* idx, char* ws, const Workspace& w, cudaStream_t st, int BK = 0,
                       int kb = 0) {
  SelectParams p{};
  p.BK = BK;
  p.kb = kb;
  p.Q = static_cast<const __nv_bfloat16*>(Q);
  p.K = static_cast<const __nv_bfloat16*>(K);
  p.perm = perm;
  p.lse = lse;
  p.idx = idx;
  p.scratch = reinterpret_cast<float*>(ws + w.scores);
  p.scratch_stride = w.score_stride;
  p.BH = s.B * s.H;
  p.N = s.N;
  p.C = C;
  p.G = s.N / C;
  p.k = k;
  p.key_tiles = (s.N + 127) / 128;
  p.num_units = p.BH * p.G;
  p.scale_log2 = resolve_scale(s) * kLog2e;
  const int grid = w.sel_grid;
  alignas(64) CUtensorMap tmK;
  if (!make_row_map(&tmK, K, static_cast<uint64_t>(p.BH) * p.N, s.d, 128)) return MCS_ERR_CUDA;
  if (BK > 0) {
    if (s.d == 64) {
      if (C == 64) select_kernel<64, 64, true><<<grid, kSelThreads, SelectSmem<64>::BYTES, st>>>(tmK, p);
      else select_kernel<64, 128, true><<<grid, kSelThreads, SelectSmem<64>::BYTES, st>>>(tmK, p);
    } else {
      if (C == 64) select_kernel<128, 64, true><<<grid, kSelThreads, SelectSmem<128>::BYTES, st>>>(tmK, p);
      else select_kernel<128, 128, true><<<grid, kSelThreads, SelectSmem<128>::BYTES, st>>>(tmK, p);
    }
  } else if (s.d == 64) {
    if (C == 64) select_kernel<64, 64><<<grid, kSelThreads, SelectSmem<64>::BYTES, st>>>(tmK, p);
    else select_kernel<64, 128><<<grid, kSelThreads, SelectSmem<64>::BYTES, st>>>(tmK, p);
  } else {
    if (C == 64) select_kernel<128, 64><<<grid, kSelThreads, SelectSmem<128>::BYTES, st>>>(tmK, p);
    else select_kernel<128, 128><<<grid, kSelThreads, SelectSmem<128>::BYTES, st>>>(tmK, p);
  }
  return launch_status();
}

}  // namespace

using namespace mcs;

extern "C" {

int mcs_abi_version(void) { return 1; }

uint64_t mcs_set_attn_wait_limit(uint64_t ns, const uint32_t* hold) {
  g_attn_hold.store(hold);
  return g_attn_wait_ns.exchange(ns == 0 ? kWaitLimitNs : ns);
}

const char* mcs_status_string(mcs_status s) {
  switch (s) {
    case MCS_OK: return "MCS_OK";
    case MCS_ERR_INVALID_ARG: return "MCS_ERR_INVALID_ARG: null pointer or size out of range";
    case MCS_ERR_SHAPE: return "MCS_ERR_SHAPE: unsupported d or C, N not a multiple of C, or N too large";
    case MCS_ERR_DTYPE_ALIGN: return "MCS_ERR_DTYPE_ALIGN: tensor or workspace pointer misaligned";
    case MCS_ERR_UNSUPPORTED_ARCH: return "MCS_ERR_UNSUPPORTED_ARCH: needs compute capability 10.0 (B200)";
    case MCS_ERR_CUDA: return "MCS_ERR_CUDA: CUDA call or launch failed";
    case MCS_ERR_BAD_INDEX: return "MCS_ERR_BAD_INDEX: perm/idx entry outside [0, N)";
    case MCS_ERR_TIMEOUT: return "MCS_ERR_TIMEOUT: a kernel's bounded wait expired";
    case MCS_ERR_WORKSPACE: return "MCS_ERR_WORKSPACE: workspace missing or too small";
  }
  return "unknown mcs_status";
}

size_t mcs_workspace_size(mcs_shape s, int C, int k) {
  if (check_shape(s) != MCS_OK || check_groups(s, C) != MCS_OK || check_k(s, k) != MCS_OK) return 0;
  DeviceInfo* di = nullptr;
  if (current_device(&di) != MCS_OK) return 0;
  return layout(s, C, di->sms).total;
}

mcs_status mcs_dense_attn(mcs_shape s, const void* Q, const void* K, const void* V, void* O, float* lse,
                          void* stream) {
  mcs_status e = check_shape(s);
  if (e != MCS_OK) return e;
  if (!Q || !K || !V || (!O && !lse)) return MCS_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || (O && !aligned16(O)) || (lse && !aligned16(lse)))
    return MCS_ERR_DTYPE_ALIGN;
  DeviceInfo* di = nullptr;
  if ((e = current_device(&di)) != MCS_OK) return e;
  return dense_impl(s, Q, K, V, O, lse, static_cast<cudaStream_t>(stream), di->sms);
}

mcs_status mcs_group(mcs_shape s, const void* Q, int C, int32_t* perm, void* ws, size_t ws_bytes, void* stream) {
  mcs_status e = check_shape(s);
  if (e != MCS_OK) return e;
  if ((e = check_groups(s, C)) != MCS_OK) return e;
  if (!Q || !perm) return MCS_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(perm)) return MCS_ERR_DTYPE_ALIGN;
  DeviceInfo* di = nullptr;
  if ((e = current_device(&di)) != MCS_OK) return e;
  const Workspace w = layout(s, C, di->sms);
  if (!ws || ws_bytes < w.total) return MCS_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return MCS_ERR_DTYPE_ALIGN;
  return group_impl(s, Q, C, perm, static_cast<char*>(ws), w, static_cast<cudaStream_t>(stream));
}

mcs_status mcs_select(mcs_shape s, const void* Q, const void* K, const int32_t* perm, int C, int k,
                      const float* lse, int32_t* idx, void* ws, size_t ws_bytes, void* stream) {
  mcs_status e = check_shape(s);
  if (e != MCS_OK) return e;
  if ((e = check_groups(s, C)) != MCS_OK) return e;
  if ((e = check_k(s, k)) != MCS_OK) return e;
  if (!Q || !K || !perm || !idx) return MCS_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(perm) || !aligned16(idx) || (lse && !aligned16(lse)))
    return MCS_ERR_DTYPE_ALIGN;
  DeviceInfo* di = nullptr;
  if ((e = current_device(&di)) != MCS_OK) return e;
  const Workspace w = layout(s, C, di->sms);
  if (!ws || ws_bytes < w.total) return MCS_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return MCS_ERR_DTYPE_ALIGN;
  char* wsc = static_cast<char*>(ws);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!lse) {
    float* l = reinterpret_cast<float*>(wsc + w.lse);
    // pass 1 needs V only as a valid pointer; with O = NULL nothing is stored but the LSE
    if ((e = dense_impl(s, Q, K, K, nullptr, l, st, di->sms)) != MCS_OK) return e;
    lse = l;
  }
  return select_impl(s, Q, K, perm, C, k, lse, idx, wsc, w, st);
}

mcs_status mcs_sparse_attn(mcs_shape s, const void* Q, const void* K, const void* V, const int32_t* perm, int C,
                           const int32_t* idx, int k, const void* R, void* out, void* stream) {
  mcs_status e = check_shape(s);
  if (e != MCS_OK) return e;
  if ((e = check_groups(s, C)) != MCS_OK) return e;
  if ((e = check_k(s, k)) != MCS_OK) return e;
  if (!Q || !K || !V || !perm || !idx || !out) return MCS_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(perm) || !aligned16(idx) ||
      (R && !aligned16(R)) || !aligned16(out))
    return MCS_ERR_DTYPE_ALIGN;
  DeviceInfo* di = nullptr;
  if ((e = current_device(&di)) != MCS_OK) return e;
  return sparse_impl(s, Q, K, V, perm, C, idx, k, R, nullptr, out, false, static_cast<cudaStream_t>(stream),
                     di->sms);
}

size_t mcs_host_staging_size(mcs_shape s, int heads_per_chunk) {
  if (check_shape(s) != MCS_OK || heads_per_chunk < 1) return 0;
  const size_t hc = std::min(static_cast<size_t>(s.B) * s.H, static_cast<size_t>(heads_per_chunk));
  return 2 * 4 * hc * static_cast<size_t>(s.N) * s.d * 2;  // two slots of Q, K, V and out (bf16)
}

namespace {
// The side streams and events of mcs_sparse_attn_host, created on a device's first call and
// kept for the life of the process (one set per device), so that a call enqueues copies and
// kernels without creating any CUDA object.  The mutex is held while a call enqueues: each
// cudaStreamWaitEvent captures the event as recorded at that moment, so a later call that
// records the same events again cannot change what an earlier call waits for, and two calls
// from different threads only queue behind each other on the side streams.
struct HostPipeline {
  bool ready = false;
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, loaded[2] = {}, computed[2] = {}, copied[2] = {};
  bool init() {
    if (ready) return true;
    if (!in && cudaStreamCreateWithFlags(&in, cudaStreamNonBlocking) != cudaSuccess) return false;
    if (!out && cudaStreamCreateWithFlags(&out, cudaStreamNonBlocking) != cudaSuccess) return false;
    for (cudaEvent_t* e : {&start, &loaded[0], &loaded[1], &computed[0], &computed[1], &copied[0], &copied[1]})
      if (!*e && cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) return false;
    ready = true;
    return true;
  }
};
HostPipeline g_host_pipe[kMaxDevices];
std::mutex g_host_mu;
}  // namespace

mcs_status mcs_sparse_attn_host(mcs_shape s, const void* hQ, const void* hK, const void* hV, const int32_t* perm,
                                int C, const int32_t* idx, int k, const void* R, void* hOut, int heads_per_chunk,
                                void* staging, size_t staging_bytes, void* stream) {
  mcs_status e = check_shape(s);
  if (e != MCS_OK) return e;
  if ((e = check_groups(s, C)) != MCS_OK) return e;
  if ((e = check_k(s, k)) != MCS_OK) return e;
  if (heads_per_chunk < 1 || !hQ || !hK || !hV || !perm || !idx || !hOut) return MCS_ERR_INVALID_ARG;
  if (!aligned16(perm) || !aligned16(idx) || (R && !aligned16(R))) return MCS_ERR_DTYPE_ALIGN;
  const size_t need = mcs_host_staging_size(s, heads_per_chunk);
  if (!staging || staging_bytes < need) return MCS_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(staging) & 255u) return MCS_ERR_DTYPE_ALIGN;
  DeviceInfo* di = nullptr;
  if ((e = current_device(&di)) != MCS_OK) return e;

  const size_t BH = static_cast<size_t>(s.B) * s.H;
  const size_t hc = std::min(BH, static_cast<size_t>(heads_per_chunk));
  const size_t head_bytes = static_cast<size_t>(s.N) * s.d * 2;
  const size_t G = static_cast<size_t>(s.N / C);
  char* stage = static_cast<char*>(staging);
  auto part = [&](int slot, int which) { return stage + (static_cast<size_t>(slot) * 4 + which) * hc * head_bytes; };
  const cudaStream_t main = static_cast<cudaStream_t>(stream);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MCS_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_host_mu);
  HostPipeline& pl = g_host_pipe[dev];
  if (!pl.init()) return MCS_ERR_CUDA;
  // the side streams start after the work already on the caller's stream (an earlier user
  // of the staging buffer, or the producer of perm/idx/R)
  if (cudaEventRecord(pl.start, main) != cudaSuccess || cudaStreamWaitEvent(pl.in, pl.start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(pl.out, pl.start, 0) != cudaSuccess)
    return MCS_ERR_CUDA;
  const char* src[3] = {static_cast<const char*>(hQ), static_cast<const char*>(hK), static_cast<const char*>(hV)};
  const size_t chunks = (BH + hc - 1) / hc;
  for (size_t c = 0; c < chunks; ++c) {
    const int slot = static_cast<int>(c & 1);
    const size_t h0 = c * hc, nh = std::min(hc, BH - h0);
    const size_t off = h0 * head_bytes, bytes = nh * head_bytes;
    // host -> device: the slot's inputs are free once chunk c-2's kernel has read them
    if (c >= 2 && cudaStreamWaitEvent(pl.in, pl.computed[slot], 0) != cudaSuccess) return MCS_ERR_CUDA;
    for (int t = 0; t < 3; ++t)
      if (cudaMemcpyAsync(part(slot, t), src[t] + off, bytes, cudaMemcpyDefault, pl.in) != cudaSuccess)
        return MCS_ERR_CUDA;
    if (cudaEventRecord(pl.loaded[slot], pl.in) != cudaSuccess) return MCS_ERR_CUDA;
    // the kernel: after the inputs landed and after chunk c-2's output left the slot
    if (cudaStreamWaitEvent(main, pl.loaded[slot], 0) != cudaSuccess) return MCS_ERR_CUDA;
    if (c >= 2 && cudaStreamWaitEvent(main, pl.copied[slot], 0) != cudaSuccess) return MCS_ERR_CUDA;
    mcs_shape sub = s;
    sub.B = 1;
    sub.H = static_cast<int>(nh);
    e = sparse_impl(sub, part(slot, 0), part(slot, 1), part(slot, 2), perm + h0 * s.N, C, idx + h0 * G * k, k,
                    R ? static_cast<const char*>(R) + off : nullptr, nullptr, part(slot, 3), false, main, di->sms);
    if (e != MCS_OK) return e;
    if (cudaEventRecord(pl.computed[slot], main) != cudaSuccess) return MCS_ERR_CUDA;
    // device -> host
    if (cudaStreamWaitEvent(pl.out, pl.computed[slot], 0) != cudaSuccess) return MCS_ERR_CUDA;
    if (cudaMemcpyAsync(static_cast<char*>(hOut) + off, part(slot, 3), bytes, cudaMemcpyDefault, pl.out) !=
        cudaSuccess)
      return MCS_ERR_CUDA;
    if (cudaEventRecord(pl.copied[slot], pl.out) != cudaSuccess) return MCS_ERR_CUDA;
  }
  // work enqueued on the caller's stream after this call sees every output byte on the host
  if (cudaStreamWaitEvent(main, pl.copied[(chunks - 1) & 1], 0) != cudaSuccess) return MCS_ERR_CUDA;
  return MCS_OK;
}

mcs_status mcs_residual(mcs_shape s, const void* Q, const void* K, const void* V, const int32_t* perm, int C,
                        const int32_t* idx, int k, const void* O_full, void* R, void* stream) {
  mcs_status e = check_shape(s);
  if (e != MCS_OK) return e;
  if ((e = check_groups(s, C)) != MCS_OK) return e;
  if ((e = check_k(s, k)) != MCS_OK) return e;
  if (!Q || !K || !V || !perm || !idx || !O_full || !R) return MCS_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(perm) || !aligned16(idx) ||
      !aligned16(O_full) || !aligned16(R))
    return MCS_ERR_DTYPE_ALIGN;
  DeviceInfo* di = nullptr;
  if ((e = current_device(&di)) != MCS_OK) return e;
  return sparse_impl(s, Q, K, V, perm, C, idx, k, nullptr, O_full, R, true, static_cast<cudaStream_t>(stream),
                     di->sms);
}

mcs_status mcs_anchor(mcs_shape s, const void* Q, const void* K, const void* V, int C, int k, void* O_full,
                      int32_t* perm, int32_t* idx, void* R, void* ws, size_t ws_bytes, void* stream) {
  mcs_status e = check_shape(s);
  if (e != MCS_OK) return e;
  if ((e = check_groups(s, C)) != MCS_OK) return e;
  if ((e = check_k(s, k)) != MCS_OK) return e;
  if (!Q || !K || !V || !O_full || !perm || !idx || !R) return MCS_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O_full) || !aligned16(perm) ||
      !aligned16(idx) || !aligned16(R))
    return MCS_ERR_DTYPE_ALIGN;
  DeviceInfo* di = nullptr;
  if ((e = current_device(&di)) != MCS_OK) return e;
  const Workspace w = layout(s, C, di->sms);
  if (!ws || ws_bytes < w.total) return MCS_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return MCS_ERR_DTYPE_ALIGN;
  char* wsc = static_cast<char*>(ws);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* lse = reinterpret_cast<float*>(wsc + w.lse);
  if ((e = dense_impl(s, Q, K, V, O_full, lse, st, di->sms)) != MCS_OK) return e;
  if ((e = group_impl(s, Q, C, perm, wsc, w, st)) != MCS_OK) return e;
  if ((e = select_impl(s, Q, K, perm, C, k, lse, idx, wsc, w, st)) != MCS_OK) return e;
  return sparse_impl(s, Q, K, V, perm, C, idx, k, nullptr, O_full, R, true, st, di->sms);
}

mcs_status mcs_select_blocks(mcs_shape s, const void* Q, const void* K, const int32_t* perm, int C, int BK, int kb,
                             int method, const float* lse, int32_t* idx, void* ws, size_t ws_bytes, void* stream) {
  mcs_status e = check_shape(s);
  if (e != MCS_OK) return e;
  if ((e = check_groups(s, C)) != MCS_OK) return e;
  if (BK < 64 || BK % 16 || s.N % BK) return MCS_ERR_SHAPE;
  const int nb = s.N / BK;
  if (nb > 4096 || kb < 1 || kb > nb || (method != 0 && method != 1)) return MCS_ERR_INVALID_ARG;
  if (!Q || !K || !perm || !idx) return MCS_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(perm) || !aligned16(idx) || (lse && !aligned16(lse)))
    return MCS_ERR_DTYPE_ALIGN;
  DeviceInfo* di = nullptr;
  if ((e = current_device(&di)) != MCS_OK) return e;
  const Workspace w = layout(s, C, di->sms);
  if (!ws || ws_bytes < w.total) return MCS_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return MCS_ERR_DTYPE_ALIGN;
  char* wsc = static_cast<char*>(ws);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (method == 0) {
    if (!lse) {
      float* l = reinterpret_cast<float*>(wsc + w.lse);
      if ((e = dense_impl(s, Q, K, K, nullptr, l, st, di->sms)) != MCS_OK) return e;
      lse = l;
    }
    return select_impl(s, Q, K, perm, C, kb * BK, lse, idx, wsc, w, st, BK, kb);
  }
  // vanilla BSA: the block means live in the grouping keys' region (BH*N*8 bytes >= BH*nb*d*4
  // since BK >= 64 >= d/2)
  BsaParams p{};
  p.Q = static_cast<const __nv_bfloat16*>(Q);
  p.K = static_cast<const __nv_bfloat16*>(K);
  p.perm = perm;
  p.kbar = reinterpret_cast<float*>(wsc + w.keys);
  p.idx = idx;
  p.BH = s.B * s.H;
  p.N = s.N;
  p.C = C;
  p.G = s.N / C;
  p.d = s.d;
  p.BK = BK;
  p.nb = nb;
  p.kb = kb;
  bsa_pool_kernel<<<dim3(nb, p.BH), s.d, 0, st>>>(p);
  const size_t smem = static_cast<size_t>(s.d + 2 * nb + 16) * 4;
  bsa_select_kernel<<<dim3(p.G, p.BH), kBsaThreads, smem, st>>>(p);
  return launch_status();
}

size_t mcs_perquery_workspace_size(mcs_shape s) {
  if (check_shape(s) != MCS_OK || s.N % 16) return 0;
  DeviceInfo* di = nullptr;
  if (current_device(&di) != MCS_OK) return 0;
  return static_cast<size_t>(di->sms) * kPqWarps * static_cast<size_t>(s.N) * 4;
}

mcs_status mcs_perquery_attn(mcs_shape s, const void* Q, const void* K, const void* V, int k, void* out, void* ws,
                             size_t ws_bytes, void* stream) {
  mcs_status e = check_shape(s);
  if (e != MCS_OK) return e;
  if (s.N % 16) return MCS_ERR_SHAPE;
  if ((e = check_k(s, k)) != MCS_OK) return e;
  if (!Q || !K || !V || !out) return MCS_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(out)) return MCS_ERR_DTYPE_ALIGN;
  DeviceInfo* di = nullptr;
  if ((e = current_device(&di)) != MCS_OK) return e;
  const size_t need = static_cast<size_t>(di->sms) * kPqWarps * static_cast<size_t>(s.N) * 4;
  if (!ws || ws_bytes < need) return MCS_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return MCS_ERR_DTYPE_ALIGN;
  PerQueryParams p{};
  p.Q = static_cast<const __nv_bfloat16*>(Q);
  p.K = static_cast<const __nv_bfloat16*>(K);
  p.V = static_cast<const __nv_bfloat16*>(V);
  p.out = static_cast<__nv_bfloat16*>(out);
  p.scratch = static_cast<float*>(ws);
  p.BH = s.B * s.H;
  p.N = s.N;
  p.d = s.d;
  p.k = k;
  p.scale = resolve_scale(s);
  p.num_rows = static_cast<long long>(p.BH) * s.N;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (s.d == 64) perquery_attn_kernel<64><<<di->sms, kPqWarps * 32, 0, st>>>(p);
  else perquery_attn_kernel<128><<<di->sms, kPqWarps * 32, 0, st>>>(p);
  return launch_status();
}

size_t mcs_kmeans_workspace_size(mcs_shape s, int C) {
  if (check_shape(s) != MCS_OK || check_groups(s, C) != MCS_OK) return 0;
  const size_t BH = static_cast<size_t>(s.B) * s.H, N = s.N, G = N / C, d = s.d;
  return round_up(BH * G * d * 8, 256) + round_up(BH * N * 4, 256) + round_up(BH * G * N * 8, 256) +
         round_up(BH * N, 256);
}

mcs_status mcs_group_kmeans(mcs_shape s, const void* Q, int C, int iters, int32_t* perm, void* ws, size_t ws_bytes,
                            void* stream) {
  mcs_status e = check_shape(s);
  if (e != MCS_OK) return e;
  if ((e = check_groups(s, C)) != MCS_OK) return e;
  if (iters < 0 || iters > 1000) return MCS_ERR_INVALID_ARG;
  if (!Q || !perm) return MCS_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(perm)) return MCS_ERR_DTYPE_ALIGN;
  DeviceInfo* di = nullptr;
  if ((e = current_device(&di)) != MCS_OK) return e;
  const size_t need = mcs_kmeans_workspace_size(s, C);
  if (!ws || ws_bytes < need) return MCS_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return MCS_ERR_DTYPE_ALIGN;
  const size_t BH = static_cast<size_t>(s.B) * s.H, N = s.N, G = N / C, d = s.d;
  char* w = static_cast<char*>(ws);
  KmeansParams p{};
  p.Q = static_cast<const __nv_bfloat16*>(Q);
  p.cent = reinterpret_cast<double*>(w);
  w += round_up(BH * G * d * 8, 256);
  p.assign = reinterpret_cast<int32_t*>(w);
  w += round_up(BH * N * 4, 256);
  p.dist = reinterpret_cast<double*>(w);
  w += round_up(BH * G * N * 8, 256);
  p.taken = reinterpret_cast<unsigned char*>(w);
  p.perm = perm;
  p.BH = static_cast<int>(BH);
  p.N = s.N;
  p.C = C;
  p.G = static_cast<int>(G);
  p.d = s.d;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const dim3 gridG(p.G, p.BH), gridQ((s.N + kKmQueries - 1) / kKmQueries, p.BH);
  kmeans_init_kernel<<<gridG, s.d, 0, st>>>(p);
  for (int it = 0; it < iters; ++it) {
    if (s.d == 64) {
      kmeans_dist_kernel<64, false><<<gridQ, kKmQueries, KmeansSmem<64>::BYTES, st>>>(p);
      kmeans_update_kernel<64><<<gridG, 64, 0, st>>>(p);
    } else {
      kmeans_dist_kernel<128, false><<<gridQ, kKmQueries, KmeansSmem<128>::BYTES, st>>>(p);
      kmeans_update_kernel<128><<<gridG, 128, 0, st>>>(p);
    }
  }
  if (s.d == 64) kmeans_dist_kernel<64, true><<<gridQ, kKmQueries, KmeansSmem<64>::BYTES, st>>>(p);
  else kmeans_dist_kernel<128, true><<<gridQ, kKmQueries, KmeansSmem<128>::BYTES, st>>>(p);
  kmeans_balance_kernel<<<p.BH, 512, 0, st>>>(p);
  return launch_status();
}

mcs_status mcs_sync_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MCS_ERR_CUDA;
  uint32_t bits = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&bits, mcs::g_status, sizeof(bits)) != cudaSuccess) return MCS_ERR_CUDA;
  if (bits && cudaMemcpyToSymbol(mcs::g_status, &zero, sizeof(zero)) != cudaSuccess) return MCS_ERR_CUDA;
  if (bits & kStatusTimeout) return MCS_ERR_TIMEOUT;
  if (bits & kStatusBadIndex) return MCS_ERR_BAD_INDEX;
  return MCS_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------------------
// Selection without any device allocation: the per-CTA score scratch of the selection kernel
// lives in this fixed array instead of a caller-provided workspace.
// ---------------------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchFloats = size_t(4) << 20;  // 16 MiB of fp32 scores
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

void* g_noalloc_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device, looked up once per device.
mcs_status noalloc_scratch(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MCS_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return MCS_ERR_CUDA;
    g_noalloc_addr[dev] = p;
  }
  *out = static_cast<float*>(g_noalloc_addr[dev]);
  return MCS_OK;
}

}  // namespace

extern "C" mcs_status mcs_select_noalloc(mcs_shape s, const void* Q, const void* K, const int32_t* perm, int C,
                                         int k, const float* lse, int32_t* idx, void* stream) {
  mcs_status e = check_shape(s);
  if (e != MCS_OK) return e;
  if ((e = check_groups(s, C)) != MCS_OK) return e;
  if ((e = check_k(s, k)) != MCS_OK) return e;
  if (!Q || !K || !perm || !lse || !idx) return MCS_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(perm) || !aligned16(idx) || !aligned16(lse))
    return MCS_ERR_DTYPE_ALIGN;
  DeviceInfo* di = nullptr;
  if ((e = current_device(&di)) != MCS_OK) return e;
  const size_t stride = round_up(static_cast<size_t>(s.N), 64);
  if (2 * stride > kNoAllocScratchFloats) return MCS_ERR_WORKSPACE;  // N beyond the fixed scratch
  float* scratch = nullptr;
  if ((e = noalloc_scratch(&scratch)) != MCS_OK) return e;
  const size_t units = static_cast<size_t>(s.B) * s.H * (s.N / C);
  Workspace w{};
  w.scores = 0;
  w.score_stride = stride;
  w.sel_grid = static_cast<int>(std::min({units, static_cast<size_t>(di->sms), kNoAllocScratchFloats / (2 * stride)}));
  return select_impl(s, Q, K, perm, C, k, lse, idx, reinterpret_cast<char*>(scratch), w,
                     static_cast<cudaStream_t>(stream));
}
