// Host side of libar_attn.so: argument validation, workspace layout, TMA
// tensor maps and kernel launches behind the C ABI declared in ar_attn.h.
#include "ar_attn.h"

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cctype>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>
#include <vector>

#include "aux.cuh"
#include "bwd.cuh"
#include "dq.cuh"
#include "fwd.cuh"
#include "sm100.cuh"

namespace {

constexpr int kD = 128;  // the head dimension of the RoPE and no-alloc paths; the others take 64 or 128
constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  int status = AR_OK;  // AR_OK or AR_ERR_DEVICE / AR_ERR_CUDA
  int sms = 0;
  int prep_blocks = 1;  // resident 256-thread blocks of the delta pre-pass per SM
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
// Limit of every device-side wait in the kernels launched from now on.
std::atomic<unsigned long long> g_wait_ns{ar::kWaitLimitNs};

// Checks the current device once: compute capability 10.0, kernel attributes.
using FwdKernel = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, ar::FwdParams);
cudaError_t fwd_attr(FwdKernel f) {
  return cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, ar::fwd::kSmemBytes);
}
bool fwd_regs_ok(FwdKernel f) {
  cudaFuncAttributes a;
  return cudaFuncGetAttributes(&a, f) == cudaSuccess && a.numRegs == ar::fwd::kLaunchRegs;
}
using BwdKernel = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, ar::BwdParams);
cudaError_t bwd_attr(BwdKernel f) {
  return cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, ar::bwd::kSmemBytes);
}

int device_setup(int* sms_out, int* prep_blocks_out = nullptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return AR_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return AR_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    d.ready = true;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      d.status = AR_ERR_CUDA;
    } else if (major != 10 || minor != 0) {
      d.status = AR_ERR_DEVICE;
    } else if (fwd_attr(ar::fwd::fwd_kernel<true, false>) != cudaSuccess ||
               fwd_attr(ar::fwd::fwd_kernel<false, false>) != cudaSuccess ||
               fwd_attr(ar::fwd::fwd_kernel<true, true>) != cudaSuccess ||
               fwd_attr(ar::fwd::fwd_kernel<false, true>) != cudaSuccess ||
               fwd_attr(ar::fwd::fwd_kernel<true, false, true>) != cudaSuccess ||
               fwd_attr(ar::fwd::fwd_kernel<false, false, true>) != cudaSuccess ||
               fwd_attr(ar::fwd::fwd_kernel<true, false, false, 64>) != cudaSuccess ||
               fwd_attr(ar::fwd::fwd_kernel<false, false, false, 64>) != cudaSuccess ||
               bwd_attr(ar::bwd::bwd_kernel<0>) != cudaSuccess || bwd_attr(ar::bwd::bwd_kernel<1>) != cudaSuccess ||
               bwd_attr(ar::bwd::bwd_kernel<3>) != cudaSuccess || bwd_attr(ar::bwd::bwd_kernel<0, 64>) != cudaSuccess ||
               cudaFuncSetAttribute(ar::dqk::dq_kernel<false, 64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    ar::dqk::kSmemBytes) != cudaSuccess ||
               cudaFuncSetAttribute(ar::dqk::dq_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    ar::dqk::kSmemBytes) != cudaSuccess ||
               cudaFuncSetAttribute(ar::dqk::dq_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    ar::dqk::kSmemBytes) != cudaSuccess) {
      d.status = AR_ERR_CUDA;
    }
    if (d.status == AR_OK) {
      // The forward moves registers between warpgroups with setmaxnreg; its split
      // is sized for exactly ar::fwd::kLaunchRegs registers per thread at launch,
      // so refuse any other build rather than launch a kernel whose register raise
      // cannot be met.  The backward kernel is checked for its own budget.
      if (!fwd_regs_ok(ar::fwd::fwd_kernel<true, false>) || !fwd_regs_ok(ar::fwd::fwd_kernel<false, false>) ||
          !fwd_regs_ok(ar::fwd::fwd_kernel<true, true>) || !fwd_regs_ok(ar::fwd::fwd_kernel<false, true>) ||
          !fwd_regs_ok(ar::fwd::fwd_kernel<true, false, true>) ||
          !fwd_regs_ok(ar::fwd::fwd_kernel<false, false, true>) ||
          !fwd_regs_ok(ar::fwd::fwd_kernel<true, false, false, 64>) ||
          !fwd_regs_ok(ar::fwd::fwd_kernel<false, false, false, 64>))
        d.status = AR_ERR_CUDA;
      for (BwdKernel f : {ar::bwd::bwd_kernel<0>, ar::bwd::bwd_kernel<1>, ar::bwd::bwd_kernel<3>,
                          ar::bwd::bwd_kernel<0, 64>}) {
        cudaFuncAttributes ba;
        if (cudaFuncGetAttributes(&ba, f) != cudaSuccess || ba.numRegs != ar::bwd::kLaunchRegs) d.status = AR_ERR_CUDA;
      }
    }
    if (d.status == AR_OK &&
        (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.prep_blocks, ar::bwd_prep_kernel<128>, 256, 0) !=
             cudaSuccess ||
         d.prep_blocks < 1))
      d.status = AR_ERR_CUDA;
    if (!g_encode && d.status == AR_OK) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) !=
              cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        d.status = AR_ERR_CUDA;
      else
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
  }
  if (d.status != AR_OK) {
    cudaGetLastError();  // clear any sticky-free error left by the attribute calls
    return d.status;
  }
  *sms_out = d.sms;
  if (prep_blocks_out) *prep_blocks_out = d.prep_blocks;
  return AR_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Head dimensions 64 and 128 (d128_only: the paths built for 128 alone).
int check_shape(int B, int T, int H, int D, bool d128_only = false) {
  if (B <= 0 || T <= 0 || H <= 0) return AR_ERR_SHAPE;
  if (D != 128 && (d128_only || D != 64)) return AR_ERR_UNSUPPORTED;
  const long long T_pad = (T + 127LL) / 128 * 128;
  // all element indices must fit comfortably in 63 bits and unit counts in int
  if ((long long)B * H * T_pad > (1LL << 31) / 2) return AR_ERR_SHAPE;
  if ((long long)B * T * H * D > (1LL << 40)) return AR_ERR_SHAPE;
  return AR_OK;
}

int check_args(float eps, float scale) {
  if (!std::isfinite(eps) || eps < 0.f) return AR_ERR_ARG;
  if (!std::isfinite(scale) || scale <= 0.f) return AR_ERR_ARG;
  return AR_OK;
}

int effective_window(int window, int T) { return (window < 0 || window >= T - 1) ? T : window; }

// Grouped K/V heads: Hkv divides H (Hkv = H is multi-head attention).
int check_kv_heads(int H, int Hkv) { return (Hkv >= 1 && Hkv <= H && H % Hkv == 0) ? AR_OK : AR_ERR_SHAPE; }

// [B, T, H, D] bf16 viewed as a 4-D tensor (d, h, t, b); boxes of 64 x 1 x 128 x 1
// land as 128 rows of 128 bytes with the 128-byte swizzle the MMA descriptors
// expect (D / 64 boxes per tile).
int make_map(CUtensorMap* m, const void* base, int B, int T, int H, int D = kD) {
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)T * H * D * 2};
  cuuint32_t box[4] = {64, 1, 128, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? AR_OK : AR_ERR_CUDA;
}

ar::FwdParams fwd_params(void* o, float* lse, const float* ck, int B, int T, int H, int Hkv, int window,
                         float eps, float scale, int D = kD) {
  ar::FwdParams p;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.rcos = p.rsin = nullptr;
  p.lse = lse;
  p.ck = ck;
  p.B = B;
  p.T = T;
  p.H = H;
  p.grp = H / Hkv;
  p.T_pad = (T + 127) / 128 * 128;
  p.w = effective_window(window, T);
  p.nqp = (T + 255) / 256;
  p.n_units = B * H * p.nqp;
  p.eps = eps;
  p.bound = scale * (float)D * 1.4426950408889634f;
  p.cscale = scale * 1.4426950408889634f;
  p.wide = aligned(o, 32);
  p.wait_ns = g_wait_ns.load();
  return p;
}

// The forward with the fixed softmax offset when the logit bound allows it
// (see fwd.cuh), else the running-max forward; key factors computed in the
// kernel, or (ck_global) read from p.ck; rope_q: Q tiles rotated in the kernel.
void launch_fwd(int grid, cudaStream_t s, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                const ar::FwdParams& p, bool ck_global, bool rope_q = false, int D = kD) {
  using namespace ar::fwd;
  const bool fixed = p.bound <= kFixedBoundMax;
  if (D == 64 && fixed)
    fwd_kernel<true, false, false, 64><<<grid, kThreads, kSmemBytes, s>>>(tq, tk, tv, p);
  else if (D == 64)
    fwd_kernel<false, false, false, 64><<<grid, kThreads, kSmemBytes, s>>>(tq, tk, tv, p);
  else if (rope_q && fixed)
    fwd_kernel<true, false, true><<<grid, kThreads, kSmemBytes, s>>>(tq, tk, tv, p);
  else if (rope_q)
    fwd_kernel<false, false, true><<<grid, kThreads, kSmemBytes, s>>>(tq, tk, tv, p);
  else if (fixed && !ck_global)
    fwd_kernel<true, false><<<grid, kThreads, kSmemBytes, s>>>(tq, tk, tv, p);
  else if (!fixed && !ck_global)
    fwd_kernel<false, false><<<grid, kThreads, kSmemBytes, s>>>(tq, tk, tv, p);
  else if (fixed)
    fwd_kernel<true, true><<<grid, kThreads, kSmemBytes, s>>>(tq, tk, tv, p);
  else
    fwd_kernel<false, true><<<grid, kThreads, kSmemBytes, s>>>(tq, tk, tv, p);
}

size_t vec_bytes(int B, int T, int H) {
  const size_t T_pad = round_up((size_t)T, 128);
  return round_up((size_t)B * H * T_pad * sizeof(float), 256);
}

// The G buffer of the backward: one 128x128 bf16 tile (32 KB) per (query tile,
// key tile) pair of the band, per head.  nb = key tiles in a query tile's band.
constexpr size_t kGTile = 32768;
constexpr size_t kGBufferCap = size_t(1) << 30;  // heads are processed in groups whose G tiles fit in this
long long g_pairs_head(int T, int nb) {
  const long long nq = (T + 127) / 128;
  return nq <= nb ? nq * (nq + 1) / 2 : (long long)nb * (nb + 1) / 2 + (nq - nb) * nb;
}
size_t g_head_bytes(int T, int nb) { return (size_t)g_pairs_head(T, nb) * kGTile; }
// Query heads whose G tiles the workspace holds at once, sized for the widest
// band (full causal): whole groups of grp query heads (the heads that share a
// K/V head are processed by one launch), at least one group.
size_t g_heads_cap(int B, int T, int H, int grp) {
  const size_t per = g_head_bytes(T, (T + 127) / 128);
  size_t n = kGBufferCap / per / grp * grp;
  if (n < (size_t)grp) n = grp;
  const size_t bh = (size_t)B * H;
  return n < bh ? n : bh;
}
int band_tiles(int w, int T) {
  const int nq = (T + 127) / 128;
  const long long nb = ((long long)w + 127) / 128 + 1;
  return nb < nq ? (int)nb : nq;
}

// [rows, 64] bf16 viewed as 2-D; boxes of 64 x 128 land as one 128-byte-swizzled
// half of a G^T tile.
int make_g_map(CUtensorMap* m, void* base, long long rows) {
  cuuint64_t dims[2] = {64, (cuuint64_t)rows};
  cuuint64_t strides[1] = {128};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? AR_OK : AR_ERR_CUDA;
}

// ---------------------------------------------------------------- kernel timing
struct TimingRec {
  int kind;
  cudaEvent_t a, b;
};
struct Timing {
  std::mutex mu;
  bool on = false;
  std::vector<TimingRec> recs;
  std::vector<cudaEvent_t> pool;
} g_timing;

cudaEvent_t timing_event() {
  if (!g_timing.pool.empty()) {
    cudaEvent_t e = g_timing.pool.back();
    g_timing.pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

// Brackets one launch with events when timing is enabled.
struct KernelTimer {
  int kind;
  cudaStream_t s;
  cudaEvent_t a = nullptr;
  KernelTimer(int kind_, cudaStream_t s_) : kind(kind_), s(s_) {
    std::lock_guard<std::mutex> lock(g_timing.mu);
    if (!g_timing.on) return;
    a = timing_event();
    if (a) cudaEventRecord(a, s);
  }
  void stop() {
    if (!a) return;
    std::lock_guard<std::mutex> lock(g_timing.mu);
    cudaEvent_t b = timing_event();
    if (!b) return;
    cudaEventRecord(b, s);
    g_timing.recs.push_back({kind, a, b});
    a = nullptr;
  }
};

int prep_grid(long long rows, int sms) {
  long long blocks = (rows + 15) / 16;  // 16 rows per 256-thread block
  const long long cap = (long long)sms * 16;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  return (int)blocks;
}

// The memory-bound passes: 64 rows per 256-thread block and iteration (two per
// lane group of 8), as many blocks as are resident on the GPU at once, looping
// over the rows.
int bwd_prep_grid(long long rows, int sms, int per_sm) {
  long long blocks = (rows + 63) / 64;
  const long long cap = (long long)sms * per_sm;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  return (int)blocks;
}

}  // namespace

extern "C" {

size_t ar_attn_bwd_gqa_workspace_bytes(int B, int T, int H, int Hkv, int D) {
  if (check_shape(B, T, H, D) != AR_OK || check_kv_heads(H, Hkv) != AR_OK) return 0;
  return 3 * vec_bytes(B, T, H) + g_heads_cap(B, T, H, H / Hkv) * g_head_bytes(T, (T + 127) / 128);
}

size_t ar_attn_bwd_workspace_bytes(int B, int T, int H, int D) { return ar_attn_bwd_gqa_workspace_bytes(B, T, H, H, D); }

int ar_attn_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse, int B, int T, int H, int Hkv,
                    int D, int window, float eps, float scale, void* stream) {
  if (!q || !k || !v || !o) return AR_ERR_NULL;  // lse may be NULL: not stored
  int st = check_shape(B, T, H, D);
  if (st != AR_OK) return st;
  if ((st = check_kv_heads(H, Hkv)) != AR_OK) return st;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
    return AR_ERR_ALIGN;
  if ((st = check_args(eps, scale)) != AR_OK) return st;
  int sms = 0;
  if ((st = device_setup(&sms)) != AR_OK) return st;

  CUtensorMap tq, tk, tv;
  if (make_map(&tq, q, B, T, H, D) != AR_OK || make_map(&tk, k, B, T, Hkv, D) != AR_OK ||
      make_map(&tv, v, B, T, Hkv, D) != AR_OK)
    return AR_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const ar::FwdParams p = fwd_params(o, lse, nullptr, B, T, H, Hkv, window, eps, scale, D);
  const int grid = p.n_units < sms ? p.n_units : sms;
  {
    KernelTimer t(AR_KERNEL_FWD, s);
    launch_fwd(grid, s, tq, tk, tv, p, false, false, D);
    t.stop();
  }
  return cudaGetLastError() == cudaSuccess ? AR_OK : AR_ERR_CUDA;
}

size_t ar_attn_fwd_rope_workspace_bytes(int B, int T, int Hkv, int D, int with_ve) {
  if (check_shape(B, T, Hkv, D, true) != AR_OK) return 0;
  return round_up((size_t)B * T * Hkv * kD * 2, 256) * (with_ve ? 2 : 1);
}

int ar_attn_fwd_rope(const void* q, const void* k, const void* v, void* o, float* lse, const void* rope_cos,
                     const void* rope_sin, int rope_rows, const void* ve, const void* ve_gate, int B, int T, int H,
                     int Hkv, int D, int window, float eps, float scale, void* workspace, size_t workspace_bytes,
                     void* stream) {
  if (!q || !k || !v || !o || !rope_cos || !rope_sin) return AR_ERR_NULL;  // lse may be NULL: not stored
  if ((ve == nullptr) != (ve_gate == nullptr)) return AR_ERR_NULL;
  int st = check_shape(B, T, H, D, true);
  if (st != AR_OK) return st;
  if ((st = check_kv_heads(H, Hkv)) != AR_OK) return st;
  if (rope_rows < T) return AR_ERR_SHAPE;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4) ||
      !aligned(rope_cos, 16) || !aligned(rope_sin, 16) || !aligned(ve, 16) || !aligned(ve_gate, 2))
    return AR_ERR_ALIGN;
  if ((st = check_args(eps, scale)) != AR_OK) return st;
  const size_t need = ar_attn_fwd_rope_workspace_bytes(B, T, Hkv, D, ve != nullptr);
  if (workspace && workspace_bytes < need) return AR_ERR_WORKSPACE;
  if (workspace && !aligned(workspace, 256)) return AR_ERR_ALIGN;
  int sms = 0, prep_blocks = 1;
  if ((st = device_setup(&sms, &prep_blocks)) != AR_OK) return st;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* ws = workspace;
  if (!ws && cudaMallocAsync(&ws, need, s) != cudaSuccess) return AR_ERR_CUDA;
  // the rotated k and the mixed v, once per layer (a K or V tile is read by every
  // unit whose band covers it); Q is rotated in the kernel's tiles
  __nv_bfloat16* kr = static_cast<__nv_bfloat16*>(ws);
  __nv_bfloat16* vm = kr + round_up((size_t)B * T * Hkv * kD * 2, 256) / 2;
  const __nv_bfloat16* rc = static_cast<const __nv_bfloat16*>(rope_cos);
  const __nv_bfloat16* rs = static_cast<const __nv_bfloat16*>(rope_sin);
  {
    KernelTimer t(AR_KERNEL_ROPE_PREP, s);
    const long long prows = (long long)B * T * Hkv * (ve ? 2 : 1);
    ar::rope_ve_prep_kernel<<<bwd_prep_grid(prows, sms, prep_blocks), 256, 0, s>>>(
        nullptr, static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v),
        static_cast<const __nv_bfloat16*>(ve), static_cast<const __nv_bfloat16*>(ve_gate), rc, rs, nullptr, kr, vm,
        B, T, H, Hkv);
    t.stop();
  }
  CUtensorMap tq, tk, tv;
  if (make_map(&tq, q, B, T, H) != AR_OK || make_map(&tk, kr, B, T, Hkv) != AR_OK ||
      make_map(&tv, ve ? static_cast<const void*>(vm) : v, B, T, Hkv) != AR_OK) {
    if (!workspace) cudaFreeAsync(ws, s);
    return AR_ERR_CUDA;
  }
  ar::FwdParams p = fwd_params(o, lse, nullptr, B, T, H, Hkv, window, eps, scale);
  p.rcos = rc;
  p.rsin = rs;
  const int grid = p.n_units < sms ? p.n_units : sms;
  {
    KernelTimer t(AR_KERNEL_FWD, s);
    launch_fwd(grid, s, tq, tk, tv, p, false, true);
    t.stop();
  }
  cudaError_t e = cudaGetLastError();
  if (!workspace) cudaFreeAsync(ws, s);
  return e == cudaSuccess ? AR_OK : AR_ERR_CUDA;
}

int ar_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int T, int H, int D,
                int window, float eps, float scale, void* stream) {
  return ar_attn_fwd_gqa(q, k, v, o, lse, B, T, H, H, D, window, eps, scale, stream);
}

}  // extern "C"

namespace {

// The RoPE / value-embedding arguments of the backward (NULL pointers: off).
struct RopeArgs {
  const __nv_bfloat16 *rcos = nullptr, *rsin = nullptr, *ve = nullptr, *vg = nullptr;
  __nv_bfloat16* dve = nullptr;
  float* dg = nullptr;
  // the forward's workspace for the same inputs: its rotated k (and mixed v),
  // used instead of forming them again (NULL: the pre-pass forms them)
  const __nv_bfloat16* saved = nullptr;
};

// Extra workspace of the RoPE path: the rotated q and k and (with a value
// embedding) the mixed v, bf16, after the G buffer.
size_t rope_bytes(int B, int T, int H, int Hkv, bool with_ve) {
  const size_t kvb = round_up((size_t)B * T * Hkv * kD * 2, 256);
  return round_up((size_t)B * T * H * kD * 2, 256) + kvb * (with_ve ? 2 : 1);
}

int bwd_run(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse, void* dq,
            void* dk, void* dv, int B, int T, int H, int Hkv, int D, int window, float eps, float scale,
            void* workspace, size_t need, void* stream, const RopeArgs* ra) {
  int sms = 0, prep_blocks = 1;
  int st = device_setup(&sms, &prep_blocks);
  if (st != AR_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* ws = workspace;
  if (!ws && cudaMallocAsync(&ws, need, s) != cudaSuccess) return AR_ERR_CUDA;

  const int grp = H / Hkv;
  const int T_pad = (T + 127) / 128 * 128;
  char* w8 = static_cast<char*>(ws);
  const size_t vb = vec_bytes(B, T, H);
  float* lse2 = reinterpret_cast<float*>(w8);
  float* delta = reinterpret_cast<float*>(w8 + vb);
  float* rq = reinterpret_cast<float*>(w8 + 2 * vb);
  char* gbuf = w8 + 3 * vb;
  const long long rows = (long long)B * T * H;
  const int pro = ra ? (ra->ve ? 3 : 1) : 0;

  // the operands the backward kernels read: q, k, v themselves, or (RoPE path)
  // the rotated q, k and mixed v the pre-pass writes after the G buffer
  const void *qx = q, *kx = k, *vx = v;
  if (ra) {
    char* r8 = gbuf + g_heads_cap(B, T, H, grp) * g_head_bytes(T, (T + 127) / 128);
    __nv_bfloat16* qr = reinterpret_cast<__nv_bfloat16*>(r8);
    __nv_bfloat16* kr = reinterpret_cast<__nv_bfloat16*>(r8 + round_up((size_t)B * T * H * kD * 2, 256));
    __nv_bfloat16* vm = kr + round_up((size_t)B * T * Hkv * kD * 2, 256) / 2;
    if (ra->saved) {
      // the forward's pre-pass output: rotated k at the start, mixed v after it
      kr = const_cast<__nv_bfloat16*>(ra->saved);
      vm = kr + round_up((size_t)B * T * Hkv * kD * 2, 256) / 2;
    }
    const long long prows = rows + (ra->saved ? 0 : (long long)B * T * Hkv * (ra->ve ? 2 : 1));
    KernelTimer t(AR_KERNEL_ROPE_PREP, s);
    ar::rope_ve_prep_kernel<<<bwd_prep_grid(prows, sms, prep_blocks), 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(q), ra->saved ? nullptr : static_cast<const __nv_bfloat16*>(k),
        static_cast<const __nv_bfloat16*>(v), ra->saved ? nullptr : ra->ve, ra->vg, ra->rcos, ra->rsin, qr, kr, vm,
        B, T, H, Hkv);
    t.stop();
    qx = qr;
    kx = kr;
    if (ra->ve) vx = vm;
  }
  CUtensorMap tq, tk, tv, tdo;
  if (make_map(&tq, qx, B, T, H, D) != AR_OK || make_map(&tk, kx, B, T, Hkv, D) != AR_OK ||
      make_map(&tv, vx, B, T, Hkv, D) != AR_OK || make_map(&tdo, dO, B, T, H, D) != AR_OK) {
    if (!workspace) cudaFreeAsync(ws, s);
    return AR_ERR_CUDA;
  }

  {
    KernelTimer t(AR_KERNEL_BWD_PREP, s);
    const int wide = aligned(qx, 32) && aligned(o, 32) && aligned(dO, 32);
    if (D == 64)
      ar::bwd_prep_kernel<64><<<bwd_prep_grid(rows, sms, prep_blocks), 256, 0, s>>>(
          static_cast<const __nv_bfloat16*>(qx), static_cast<const __nv_bfloat16*>(o),
          static_cast<const __nv_bfloat16*>(dO), lse, lse2, delta, rq, B, T, H, T_pad, eps, wide);
    else
      ar::bwd_prep_kernel<128><<<bwd_prep_grid(rows, sms, prep_blocks), 256, 0, s>>>(
          static_cast<const __nv_bfloat16*>(qx), static_cast<const __nv_bfloat16*>(o),
          static_cast<const __nv_bfloat16*>(dO), lse, lse2, delta, rq, B, T, H, T_pad, eps, wide);
    t.stop();
  }
  const int w = effective_window(window, T);
  const int nk = (T + 127) / 128;
  const int nb = band_tiles(w, T);
  const long long ph = g_pairs_head(T, nb);
  // K/V heads per launch: as many whole groups as the G buffer holds for this window
  const long long cap_tiles = (long long)g_heads_cap(B, T, H, grp) * g_pairs_head(T, nk);
  const int BKV = B * Hkv;
  const int kpl_max = (int)std::min<long long>(BKV, std::max<long long>(1, cap_tiles / (ph * grp)));
  const int n_groups = (BKV + kpl_max - 1) / kpl_max;
  const int kpl = (BKV + n_groups - 1) / n_groups;  // equal launches
  CUtensorMap tg;
  if (make_g_map(&tg, gbuf, 2 * (long long)kpl * grp * ph * 128) != AR_OK) {
    if (!workspace) cudaFreeAsync(ws, s);
    return AR_ERR_CUDA;
  }
  for (int bk0 = 0; bk0 < BKV; bk0 += kpl) {
    const int n_bk = std::min(kpl, BKV - bk0);
    ar::BwdParams p;
    p.dk = static_cast<__nv_bfloat16*>(dk);
    p.dv = static_cast<__nv_bfloat16*>(dv);
    p.k = static_cast<const __nv_bfloat16*>(kx);
    p.lse2 = lse2;
    p.delta = delta;
    p.rq = rq;
    p.rcos = ra ? ra->rcos : nullptr;
    p.rsin = ra ? ra->rsin : nullptr;
    p.ve = ra ? ra->ve : nullptr;
    p.vg = ra ? ra->vg : nullptr;
    p.dve = ra ? ra->dve : nullptr;
    p.dg = ra ? ra->dg : nullptr;
    p.B = B;
    p.T = T;
    p.H = H;
    p.T_pad = T_pad;
    p.Hkv = Hkv;
    p.grp = grp;
    p.w = w;
    p.nk = nk;
    p.n_units = n_bk * nk;
    p.bh0 = bk0;
    p.n_bh = n_bk;
    p.nb = nb;
    p.pairs_head = (int)ph;
    p.eps = eps;
    p.scale = scale;
    p.wide = aligned(dk, 32) && aligned(dv, 32) && (p.dve == nullptr || aligned(p.dve, 32));
    p.wide_k = aligned(kx, 32);
    p.wide_ve = p.ve != nullptr && aligned(p.ve, 32);
    p.wait_ns = g_wait_ns.load();
    {
      KernelTimer t(AR_KERNEL_BWD, s);
      const int grid = std::min(p.n_units, sms);
      if (D == 64)
        ar::bwd::bwd_kernel<0, 64><<<grid, ar::bwd::kThreads, ar::bwd::kSmemBytes, s>>>(tq, tk, tv, tdo, tg, p);
      else if (pro == 0)
        ar::bwd::bwd_kernel<0><<<grid, ar::bwd::kThreads, ar::bwd::kSmemBytes, s>>>(tq, tk, tv, tdo, tg, p);
      else if (pro == 1)
        ar::bwd::bwd_kernel<1><<<grid, ar::bwd::kThreads, ar::bwd::kSmemBytes, s>>>(tq, tk, tv, tdo, tg, p);
      else
        ar::bwd::bwd_kernel<3><<<grid, ar::bwd::kThreads, ar::bwd::kSmemBytes, s>>>(tq, tk, tv, tdo, tg, p);
      t.stop();
    }
    ar::DqParams d;
    d.q = static_cast<const __nv_bfloat16*>(qx);
    d.rcos = p.rcos;
    d.rsin = p.rsin;
    d.dq = static_cast<__nv_bfloat16*>(dq);
    d.B = B;
    d.T = T;
    d.H = H;
    d.grp = grp;
    d.w = w;
    d.nq = nk;
    d.n_units = n_bk * grp * nk;  // units of one query tile of one query head
    d.bh0 = bk0 * grp;            // the query heads of K/V heads bk0 .. bk0 + n_bk - 1
    d.n_bh = n_bk * grp;
    d.nb = nb;
    d.pairs_head = (int)ph;
    d.eps = eps;
    d.scale = scale;
    d.wide = aligned(dq, 32);
    d.wide_q = aligned(qx, 32);
    d.wait_ns = p.wait_ns;
    {
      KernelTimer t(AR_KERNEL_DQ, s);
      const int grid = std::min(d.n_units, sms);
      if (D == 64)
        ar::dqk::dq_kernel<false, 64><<<grid, ar::dqk::kThreads, ar::dqk::kSmemBytes, s>>>(tg, tk, d);
      else if (ra)
        ar::dqk::dq_kernel<true><<<grid, ar::dqk::kThreads, ar::dqk::kSmemBytes, s>>>(tg, tk, d);
      else
        ar::dqk::dq_kernel<false><<<grid, ar::dqk::kThreads, ar::dqk::kSmemBytes, s>>>(tg, tk, d);
      t.stop();
    }
  }
  cudaError_t e = cudaGetLastError();
  if (!workspace) cudaFreeAsync(ws, s);
  return e == cudaSuccess ? AR_OK : AR_ERR_CUDA;
}

}  // namespace

extern "C" {

int ar_attn_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                    void* dq, void* dk, void* dv, int B, int T, int H, int Hkv, int D, int window, float eps,
                    float scale, void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !o || !dO || !lse || !dq || !dk || !dv) return AR_ERR_NULL;
  int st = check_shape(B, T, H, D);
  if (st != AR_OK) return st;
  if ((st = check_kv_heads(H, Hkv)) != AR_OK) return st;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(dO, 16) ||
      !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(lse, 4))
    return AR_ERR_ALIGN;
  if ((st = check_args(eps, scale)) != AR_OK) return st;
  const size_t need = ar_attn_bwd_gqa_workspace_bytes(B, T, H, Hkv, D);
  if (workspace && workspace_bytes < need) return AR_ERR_WORKSPACE;
  if (workspace && !aligned(workspace, 256)) return AR_ERR_ALIGN;
  return bwd_run(q, k, v, o, dO, lse, dq, dk, dv, B, T, H, Hkv, D, window, eps, scale, workspace, need, stream,
                 nullptr);
}

size_t ar_attn_bwd_rope_workspace_bytes(int B, int T, int H, int Hkv, int D, int with_ve) {
  if (D != kD) return 0;
  const size_t base = ar_attn_bwd_gqa_workspace_bytes(B, T, H, Hkv, D);
  return base ? base + rope_bytes(B, T, H, Hkv, with_ve != 0) : 0;
}

int ar_attn_bwd_rope(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                     const void* rope_cos, const void* rope_sin, int rope_rows, const void* ve, const void* ve_gate,
                     void* dq, void* dk, void* dv, void* dve, float* dgate, int B, int T, int H, int Hkv, int D,
                     int window, float eps, float scale, void* workspace, size_t workspace_bytes, void* stream) {
  return ar_attn_bwd_rope_saved(q, k, v, o, dO, lse, rope_cos, rope_sin, rope_rows, ve, ve_gate, dq, dk, dv, dve,
                                dgate, B, T, H, Hkv, D, window, eps, scale, nullptr, workspace, workspace_bytes,
                                stream);
}

int ar_attn_bwd_rope_saved(const void* q, const void* k, const void* v, const void* o, const void* dO,
                           const float* lse, const void* rope_cos, const void* rope_sin, int rope_rows,
                           const void* ve, const void* ve_gate, void* dq, void* dk, void* dv, void* dve,
                           float* dgate, int B, int T, int H, int Hkv, int D, int window, float eps, float scale,
                           const void* saved, void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !o || !dO || !lse || !dq || !dk || !dv || !rope_cos || !rope_sin) return AR_ERR_NULL;
  const bool with_ve = ve != nullptr;
  if (with_ve && (!ve_gate || !dve || !dgate)) return AR_ERR_NULL;
  if (!with_ve && (ve_gate || dve || dgate)) return AR_ERR_NULL;
  int st = check_shape(B, T, H, D, true);
  if (st != AR_OK) return st;
  if ((st = check_kv_heads(H, Hkv)) != AR_OK) return st;
  if (rope_rows < T) return AR_ERR_SHAPE;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(dO, 16) ||
      !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(lse, 4) || !aligned(rope_cos, 16) ||
      !aligned(rope_sin, 16) || !aligned(ve, 16) || !aligned(ve_gate, 2) || !aligned(dve, 16) ||
      !aligned(dgate, 4))
    return AR_ERR_ALIGN;
  if ((st = check_args(eps, scale)) != AR_OK) return st;
  const size_t need = ar_attn_bwd_rope_workspace_bytes(B, T, H, Hkv, D, with_ve);
  if (workspace && workspace_bytes < need) return AR_ERR_WORKSPACE;
  if (workspace && !aligned(workspace, 256)) return AR_ERR_ALIGN;
  if (saved && !aligned(saved, 256)) return AR_ERR_ALIGN;
  RopeArgs ra;
  ra.saved = static_cast<const __nv_bfloat16*>(saved);
  ra.rcos = static_cast<const __nv_bfloat16*>(rope_cos);
  ra.rsin = static_cast<const __nv_bfloat16*>(rope_sin);
  ra.ve = static_cast<const __nv_bfloat16*>(ve);
  ra.vg = static_cast<const __nv_bfloat16*>(ve_gate);
  ra.dve = static_cast<__nv_bfloat16*>(dve);
  ra.dg = dgate;
  return bwd_run(q, k, v, o, dO, lse, dq, dk, dv, B, T, H, Hkv, D, window, eps, scale, workspace, need, stream,
                 &ra);
}

int ar_attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                void* dq, void* dk, void* dv, int B, int T, int H, int D, int window, float eps, float scale,
                void* workspace, size_t workspace_bytes, void* stream) {
  return ar_attn_bwd_gqa(q, k, v, o, dO, lse, dq, dk, dv, B, T, H, H, D, window, eps, scale, workspace,
                         workspace_bytes, stream);
}

int ar_attn_sync_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return AR_ERR_CUDA;
  int flag = 0;
  if (cudaMemcpyFromSymbol(&flag, ar::g_status, sizeof(int)) != cudaSuccess) return AR_ERR_CUDA;
  if (flag != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(ar::g_status, &zero, sizeof(int)) != cudaSuccess) return AR_ERR_CUDA;
    return (flag & ar::DEV_LAYOUT) ? AR_ERR_LAYOUT : AR_ERR_TIMEOUT;
  }
  return AR_OK;
}

const char* ar_attn_strerror(int status) {
  switch (status) {
    case AR_OK: return "ok";
    case AR_ERR_NULL: return "a required pointer is NULL";
    case AR_ERR_SHAPE: return "invalid shape (B, T, H must be positive and within index range)";
    case AR_ERR_UNSUPPORTED: return "unsupported head dimension (only D = 128)";
    case AR_ERR_ALIGN: return "misaligned pointer (tensors need 16-byte, workspace 256-byte alignment)";
    case AR_ERR_ARG: return "invalid eps or scale (eps >= 0, scale > 0, both finite)";
    case AR_ERR_DEVICE: return "current device is not a compute capability 10.0 (B200) GPU";
    case AR_ERR_CUDA: return "a CUDA runtime call failed";
    case AR_ERR_TIMEOUT: return "a device-side wait timed out; results of the affected call are invalid";
    case AR_ERR_WORKSPACE: return "workspace smaller than the required size";
    case AR_ERR_TOO_LARGE: return "B * H * padded T exceeds the built-in scratch of ar_attn_fwd_noalloc";
    case AR_ERR_LAYOUT: return "a kernel's shared memory was not 1024-byte aligned; it did not run";
    default: return "unknown status";
  }
}

int ar_attn_layer_window(int layer, int n_layer, int seq_len, const char* pattern) {
  if (!pattern) return AR_ERR_NULL;
  const size_t len = std::strlen(pattern);
  if (len == 0 || n_layer <= 0 || seq_len <= 0 || layer < 0 || layer >= n_layer) return AR_ERR_ARG;
  if (layer == n_layer - 1) return seq_len;
  const char c = (char)std::toupper((unsigned char)pattern[layer % len]);
  if (c == 'L') return seq_len;
  if (c == 'S') return seq_len / 2;
  return AR_ERR_ARG;
}

int ar_attn_set_wait_limit_ns(unsigned long long ns) {
  g_wait_ns.store(ns == 0 ? ar::kWaitLimitNs : ns);
  return AR_OK;
}

int ar_attn_timing_enable(int on) {
  std::lock_guard<std::mutex> lock(g_timing.mu);
  if (on) {
    for (auto& r : g_timing.recs) {
      g_timing.pool.push_back(r.a);
      g_timing.pool.push_back(r.b);
    }
    g_timing.recs.clear();
  }
  g_timing.on = on != 0;
  return AR_OK;
}

int ar_attn_timing_read(double* ms, long long* count) {
  std::lock_guard<std::mutex> lock(g_timing.mu);
  double acc[AR_KERNEL_KINDS] = {};
  long long n[AR_KERNEL_KINDS] = {};
  int st = AR_OK;
  for (auto& r : g_timing.recs) {
    float t = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) {
      st = AR_ERR_CUDA;
    } else if (r.kind >= 0 && r.kind < AR_KERNEL_KINDS) {
      acc[r.kind] += t;
      n[r.kind] += 1;
    }
    g_timing.pool.push_back(r.a);
    g_timing.pool.push_back(r.b);
  }
  g_timing.recs.clear();
  for (int i = 0; i < AR_KERNEL_KINDS; ++i) {
    if (ms) ms[i] = acc[i];
    if (count) count[i] = n[i];
  }
  return st;
}

long long ar_attn_unmasked_pairs(int T, int window) {
  if (T <= 0) return 0;
  const long long w = (window < 0 || window >= T - 1) ? (long long)T : (long long)window;
  // rows i <= w see i + 1 keys, the others w + 1
  const long long n1 = (w + 1 < T) ? (w + 1) : T;
  long long total = n1 * (n1 + 1) / 2;
  total += (long long)(T - n1) * (w + 1);
  return total;
}

}  // extern "C"

// ---------------------------------------------------------------- allocation-free forward
// Scratch for ar_attn_fwd_noalloc: the per-key norm factors of up to
// AR_NOALLOC_MAX_KEYS key rows.  Compiled into the library, so it exists on
// every device that loads it, for the life of the process.  In host code the
// name is only a handle; its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) float g_noalloc_ck[AR_NOALLOC_MAX_KEYS];

namespace {
float* g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mu;

// Device address of g_noalloc_ck on the current device, looked up once.
int noalloc_scratch(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return AR_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return AR_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_ck) != cudaSuccess || ptr == nullptr) {
      cudaGetLastError();
      return AR_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = static_cast<float*>(ptr);
  }
  *out = g_noalloc_ptr[dev];
  return AR_OK;
}
}  // namespace

extern "C" int ar_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse, int B, int T,
                                   int H, int D, int window, float eps, float scale, void* stream) {
  if (!q || !k || !v || !o) return AR_ERR_NULL;  // lse may be NULL: not stored
  int st = check_shape(B, T, H, D, true);
  if (st != AR_OK) return st;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
    return AR_ERR_ALIGN;
  if ((st = check_args(eps, scale)) != AR_OK) return st;
  const int T_pad = (T + 127) / 128 * 128;
  if ((long long)B * H * T_pad > (long long)AR_NOALLOC_MAX_KEYS) return AR_ERR_TOO_LARGE;
  int sms = 0;
  if ((st = device_setup(&sms)) != AR_OK) return st;
  float* ck = nullptr;
  if ((st = noalloc_scratch(&ck)) != AR_OK) return st;

  CUtensorMap tq, tk, tv;
  if (make_map(&tq, q, B, T, H) != AR_OK || make_map(&tk, k, B, T, H) != AR_OK || make_map(&tv, v, B, T, H) != AR_OK)
    return AR_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long long rows = (long long)B * T * H;
  {
    KernelTimer t(AR_KERNEL_FWD_PREP, s);
    ar::fwd_prep_kernel<<<prep_grid(rows, sms), 256, 0, s>>>(static_cast<const __nv_bfloat16*>(k), ck, B, T, H,
                                                              T_pad, eps, scale * 1.4426950408889634f);
    t.stop();
  }
  const ar::FwdParams p = fwd_params(o, lse, ck, B, T, H, H, window, eps, scale);
  const int grid = p.n_units < sms ? p.n_units : sms;
  {
    KernelTimer t(AR_KERNEL_FWD, s);
    launch_fwd(grid, s, tq, tk, tv, p, true);
    t.stop();
  }
  return cudaGetLastError() == cudaSuccess ? AR_OK : AR_ERR_CUDA;
}
