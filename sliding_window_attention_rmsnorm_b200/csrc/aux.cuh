// Memory-bound passes around the two attention kernels.  One 128-element row
// (one token of one head) is handled by 16 lanes, 8 elements (16 bytes) each.
//
//   fwd_prep  : ck[bh, t] = rk_t * scale * log2(e), rk_t = 1/sqrt(mean_d k_td^2 + eps)
//   bwd_prep  : delta[bh, t] = sum_d dO_td o_td  (FlashAttention's backward pre-pass),
//               rq[bh, t]    = 1/sqrt(mean_d q_td^2 + eps),
//               lse2[bh, t]  = lse[bh, t] * log2(e)
// The [B*H, T_pad] vectors are zero on the padding t >= T so that every tile
// of 128 entries can be copied whole.
#pragma once
#include "sm100.cuh"

namespace ar {

__device__ __forceinline__ float half_warp_sum(float v) {
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    f[2 * e] = bf16lo(w[e]);
    f[2 * e + 1] = bf16hi(w[e]);
  }
}

// Rows are visited in memory order (b, t, h); row r is token t = (r / H) % T of
// head (b, h).  The split uses 32-bit division whenever the row count allows it
// (a 64-bit division costs several times the issue slots of the row's load).
__device__ __forceinline__ void split_row(long long r, int T, int H, int& b, int& t, int& h) {
  if (r < 0x7fffffffLL && (long long)T * H < 0x7fffffffLL) {
    const unsigned ur = (unsigned)r, bt = ur / (unsigned)H;
    h = (int)(ur - bt * (unsigned)H);
    b = (int)(bt / (unsigned)T);
    t = (int)(bt - (unsigned)b * (unsigned)T);
  } else {
    const long long bt = r / H;
    h = (int)(r - bt * H);
    b = (int)(bt / T);
    t = (int)(bt - (long long)b * T);
  }
}
__global__ void fwd_prep_kernel(const __nv_bfloat16* __restrict__ k, float* __restrict__ ck, int B, int T, int H,
                                int T_pad, float eps, float cscale) {
  const long long rows = (long long)B * T * H;
  const int sub = threadIdx.x & 15;
  const long long gstride = (long long)gridDim.x * (blockDim.x / 16);
  for (long long r = (long long)blockIdx.x * (blockDim.x / 16) + threadIdx.x / 16; r < rows; r += gstride) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(k + r * 128) + sub);
    float f[8];
    unpack8(u, f);
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) ss = fmaf(f[e], f[e], ss);
    ss = half_warp_sum(ss);
    if (sub == 0) {
      int b, t, h;
      split_row(r, T, H, b, t, h);
      ck[((long long)b * H + h) * T_pad + t] = rsqrtf(ss * (1.0f / 128.0f) + eps) * cscale;
    }
  }
  // padding entries
  const long long pads = (long long)B * H * (T_pad - T);
  for (long long x = (long long)blockIdx.x * blockDim.x + threadIdx.x; x < pads; x += (long long)gridDim.x * blockDim.x) {
    const long long bh = x / (T_pad - T);
    const int t = T + (int)(x % (T_pad - T));
    ck[bh * T_pad + t] = 0.f;
  }
}

__global__ void bwd_prep_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ o,
                                const __nv_bfloat16* __restrict__ dO, const float* __restrict__ lse,
                                float* __restrict__ lse2, float* __restrict__ delta, float* __restrict__ rq, int B,
                                int T, int H, int T_pad, float eps) {
  const long long rows = (long long)B * T * H;
  const int sub = threadIdx.x & 15;
  const long long gstride = (long long)gridDim.x * (blockDim.x / 16);
  const float kLog2e = 1.4426950408889634f;
  for (long long r = (long long)blockIdx.x * (blockDim.x / 16) + threadIdx.x / 16; r < rows; r += gstride) {
    float fq[8], fo[8], fd[8];
    unpack8(__ldg(reinterpret_cast<const uint4*>(q + r * 128) + sub), fq);
    unpack8(__ldg(reinterpret_cast<const uint4*>(o + r * 128) + sub), fo);
    unpack8(__ldg(reinterpret_cast<const uint4*>(dO + r * 128) + sub), fd);
    float ss = 0.f, dl = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      ss = fmaf(fq[e], fq[e], ss);
      dl = fmaf(fo[e], fd[e], dl);
    }
    ss = half_warp_sum(ss);
    dl = half_warp_sum(dl);
    if (sub == 0) {
      int b, t, h;
      split_row(r, T, H, b, t, h);
      const long long bh = (long long)b * H + h;
      delta[bh * T_pad + t] = dl;
      rq[bh * T_pad + t] = rsqrtf(ss * (1.0f / 128.0f) + eps);
      lse2[bh * T_pad + t] = lse[bh * T + t] * kLog2e;
    }
  }
  const long long pads = (long long)B * H * (T_pad - T);
  for (long long x = (long long)blockIdx.x * blockDim.x + threadIdx.x; x < pads; x += (long long)gridDim.x * blockDim.x) {
    const long long bh = x / (T_pad - T);
    const int t = T + (int)(x % (T_pad - T));
    delta[bh * T_pad + t] = 0.f;
    rq[bh * T_pad + t] = 0.f;
    lse2[bh * T_pad + t] = 0.f;
  }
}

}  // namespace ar
