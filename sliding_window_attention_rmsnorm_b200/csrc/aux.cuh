// Memory-bound passes around the two attention kernels.  One 128-element row
// (one token of one head) is handled by 16 lanes, 8 elements (16 bytes) each.
//
//   fwd_prep  : ck[bh, t] = rk_t * scale * log2(e), rk_t = 1/sqrt(mean_d k_td^2 + eps)
//   bwd_prep  : delta[bh, t] = sum_d dO_td o_td  (FlashAttention's backward pre-pass),
//               read 8 lanes to a row with 256-bit loads,
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

// c += sum over the 8 bf16 pairs of a and b of a_k * b_k (products exact in
// f32, one rounding per fma; the bf16 halves are read directly).
__device__ __forceinline__ void dot_bf16x8_f32(float& c0, float& c1, const uint4& a, const uint4& b) {
  const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
  for (int e = 0; e < 4; ++e)
    asm("{\n .reg .b16 al, ah, bl, bh;\n mov.b32 {al, ah}, %2;\n mov.b32 {bl, bh}, %3;\n"
        " fma.rn.f32.bf16 %0, al, bl, %0;\n fma.rn.f32.bf16 %1, ah, bh, %1;\n}"
        : "+f"(c0), "+f"(c1)
        : "r"(wa[e]), "r"(wb[e]));
}

// One row (one token of one head, D = 128 or 64 elements) per 8 lanes, D / 4
// bytes of each of q, o and dO per lane: 256-bit loads (D = 128) when the
// tensors are 32-byte aligned, 128-bit loads otherwise.  Each lane group takes
// two rows per iteration (rows r and r + half a block's stride) and issues all
// their loads before it uses any, so that enough bytes are in flight.
template <int kD>
__device__ __forceinline__ void prep_load(const __nv_bfloat16* __restrict__ x, long long base, uint4& a, uint4& b,
                                          int wide) {
  if (kD == 128) {
    ldg32B(x + base, a, b, wide);
  } else {
    a = __ldg(reinterpret_cast<const uint4*>(x + base));
    b = make_uint4(0, 0, 0, 0);
  }
}

template <int kD>
__device__ __forceinline__ void prep_row(long long r, int sub, const uint4 (&qv)[2], const uint4 (&ov)[2],
                                         const uint4 (&dv)[2], const float* __restrict__ lse,
                                         float* __restrict__ lse2, float* __restrict__ delta, float* __restrict__ rq,
                                         int T, int H, int T_pad, float eps) {
  float s0 = 0.f, s1 = 0.f, t0 = 0.f, t1 = 0.f;
#pragma unroll
  for (int h = 0; h < kD / 64; ++h) {
    fma_sq_bf16x2_f32(s0, s1, qv[h].x);
    fma_sq_bf16x2_f32(s0, s1, qv[h].y);
    fma_sq_bf16x2_f32(s0, s1, qv[h].z);
    fma_sq_bf16x2_f32(s0, s1, qv[h].w);
    dot_bf16x8_f32(t0, t1, ov[h], dv[h]);
  }
  float ss = s0 + s1, dl = t0 + t1;
#pragma unroll
  for (int m = 4; m > 0; m >>= 1) {
    ss += __shfl_xor_sync(0xffffffffu, ss, m);
    dl += __shfl_xor_sync(0xffffffffu, dl, m);
  }
  if (sub == 0) {
    int b, t, h;
    split_row(r, T, H, b, t, h);
    const long long bh = (long long)b * H + h;
    delta[bh * T_pad + t] = dl;
    rq[bh * T_pad + t] = rsqrtf(ss * (1.0f / kD) + eps);
    lse2[bh * T_pad + t] = lse[bh * T + t] * 1.4426950408889634f;
  }
}

template <int kD>
__global__ void bwd_prep_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ o,
                                const __nv_bfloat16* __restrict__ dO, const float* __restrict__ lse,
                                float* __restrict__ lse2, float* __restrict__ delta, float* __restrict__ rq, int B,
                                int T, int H, int T_pad, float eps, int wide) {
  static_assert(kD == 64 || kD == 128, "head dimension 64 or 128");
  const long long rows = (long long)B * T * H;
  const int sub = threadIdx.x & 7;
  const long long per_block = blockDim.x / 8;  // lane groups per block
  const long long gstride = (long long)gridDim.x * per_block * 2;
  for (long long r0 = (long long)blockIdx.x * per_block * 2 + threadIdx.x / 8; r0 < rows; r0 += gstride) {
    const long long r1 = r0 + per_block;
    const bool two = r1 < rows;  // uniform over the lane group
    uint4 q0[2], o0[2], d0[2], q1[2], o1[2], d1[2];
    const long long b0 = r0 * kD + sub * (kD / 8), b1 = r1 * kD + sub * (kD / 8);
    prep_load<kD>(q, b0, q0[0], q0[1], wide);
    prep_load<kD>(o, b0, o0[0], o0[1], wide);
    prep_load<kD>(dO, b0, d0[0], d0[1], wide);
    if (two) {
      prep_load<kD>(q, b1, q1[0], q1[1], wide);
      prep_load<kD>(o, b1, o1[0], o1[1], wide);
      prep_load<kD>(dO, b1, d1[0], d1[1], wide);
    }
    prep_row<kD>(r0, sub, q0, o0, d0, lse, lse2, delta, rq, T, H, T_pad, eps);
    if (two) prep_row<kD>(r1, sub, q1, o1, d1, lse, lse2, delta, rq, T, H, T_pad, eps);
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

// The pre-pass of the RoPE / value-embedding path: the rotated q and k and the
// mixed v (v + 2 sigmoid(g) ve) written out for the attention kernels, with the
// arithmetic of sm100.cuh's helpers.  Rows [0, nq) are q rows [B, T, H] (none
// when q is NULL: the forward rotates its Q tiles itself), then nk k rows and,
// when ve is given, nk v rows [B, T, Hkv] (no k or v rows when k is NULL: the
// backward given the forward's rotated k and mixed v); one row per 8 lanes.  RoPE: lane l
// rotates features 8l .. 8l+7 with their partners 64 + 8l ..; value embedding:
// lane l mixes features 16l .. 16l+15.
__global__ void rope_ve_prep_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                                    const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ ve,
                                    const __nv_bfloat16* __restrict__ vg, const __nv_bfloat16* __restrict__ rcos,
                                    const __nv_bfloat16* __restrict__ rsin, __nv_bfloat16* __restrict__ qr,
                                    __nv_bfloat16* __restrict__ kr, __nv_bfloat16* __restrict__ vm, int B, int T,
                                    int H, int Hkv) {
  const long long nq = q ? (long long)B * T * H : 0, nk = k ? (long long)B * T * Hkv : 0;
  const long long rows = nq + nk + (ve && k ? nk : 0);
  const int sub = threadIdx.x & 7;
  const long long gstride = (long long)gridDim.x * (blockDim.x / 8);
  for (long long r = (long long)blockIdx.x * (blockDim.x / 8) + threadIdx.x / 8; r < rows; r += gstride) {
    if (r < nq + nk) {
      const bool isq = r < nq;
      const long long rr = isq ? r : r - nq;
      const int t = (int)((rr / (isq ? H : Hkv)) % T);
      const __nv_bfloat16* src = (isq ? q : k) + rr * 128;
      __nv_bfloat16* dst = (isq ? qr : kr) + rr * 128;
      const uint4 x1 = __ldg(reinterpret_cast<const uint4*>(src + 8 * sub));
      const uint4 x2 = __ldg(reinterpret_cast<const uint4*>(src + 64 + 8 * sub));
      const uint4 c = __ldg(reinterpret_cast<const uint4*>(rcos + (size_t)t * 64 + 8 * sub));
      const uint4 sn = __ldg(reinterpret_cast<const uint4*>(rsin + (size_t)t * 64 + 8 * sub));
      uint4 y1, y2;
      rope_word(x1.x, x2.x, c.x, sn.x, y1.x, y2.x);
      rope_word(x1.y, x2.y, c.y, sn.y, y1.y, y2.y);
      rope_word(x1.z, x2.z, c.z, sn.z, y1.z, y2.z);
      rope_word(x1.w, x2.w, c.w, sn.w, y1.w, y2.w);
      *reinterpret_cast<uint4*>(dst + 8 * sub) = y1;
      *reinterpret_cast<uint4*>(dst + 64 + 8 * sub) = y2;
    } else {
      const long long rr = r - nq - nk;
      const uint4* src = reinterpret_cast<const uint4*>(v + rr * 128 + 16 * sub);
      uint4* dst = reinterpret_cast<uint4*>(vm + rr * 128 + 16 * sub);
      const uint4 a = __ldg(src), b = __ldg(src + 1);
      const float gate = ve_gate(vg[rr]);
      const uint4* e = reinterpret_cast<const uint4*>(ve + rr * 128 + 16 * sub);
      const uint4 ea = __ldg(e), eb = __ldg(e + 1);
      dst[0] = make_uint4(ve_mix_word(a.x, ea.x, gate), ve_mix_word(a.y, ea.y, gate), ve_mix_word(a.z, ea.z, gate),
                          ve_mix_word(a.w, ea.w, gate));
      dst[1] = make_uint4(ve_mix_word(b.x, eb.x, gate), ve_mix_word(b.y, eb.y, gate), ve_mix_word(b.z, eb.z, gate),
                          ve_mix_word(b.w, eb.w, gate));
    }
  }
}

}  // namespace ar
