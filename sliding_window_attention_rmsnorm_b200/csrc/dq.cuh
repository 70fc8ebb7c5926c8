// Query gradient of the fused QK-RMSNorm attention backward, sm_100a.
//
// dq = rq (dqhat - qhat (dqhat . qhat) / D), qhat = rq q: the RMSNorm backward
// (the same formula as for k) applied to dqhat_i = scale sum_j dS_ij khat_j,
// the attention gradient of the query (FlashAttention backward; norm(q) before
// the attention product as in the "autoresearch" README (gitee), section 7.3).
//
// The backward main kernel stores, for every (query tile, key tile) pair of the
// band, the bf16 tile G^T with G_ij = dS_ij rq_i rk_j.  Here one CTA owns one
// 128-query tile at a time (a unit) and accumulates, in TMEM,
//   acc_i = sum_j G_ij k_j = rq_i dqhat_i / scale      (raw bf16 k rows)
// over the tile's band, then finishes dq_i = scale (acc_i - c_i q_i) with
// c_i = (acc_i . q_i) / D / (mean q_i^2 + eps) and writes it as bf16.  Per key
// tile of the band the kernel streams a 32 KB G tile (from DRAM) and the 32 KB
// K tile (mostly from L2).  Units of one query tile, rather than two that share
// their K tiles, split the work into finer pieces, so the persistent CTAs end
// closer together on banded layers.
//
// CTA organisation (persistent, one CTA per SM, 224 threads):
//   warps 0-3  epilogue warpgroup: one query row per thread
//   warp 4     TMA producer of the G tiles (two 64-query halves each; 4 stages)
//   warp 5     MMA issuer
//   warp 6     TMA producer of the K tiles (3 stages)
// With the RoPE prologue (kRope) the K tiles and p.q are the rotated k and q
// the backward's pre-pass wrote, and the epilogue ends with the transposed
// rotation of the query's position: dq = R_i^T dq_rot (dq1 = d1 cos - d2 sin,
// dq2 = d1 sin + d2 cos for the halves d1, d2).
// TMEM (512 columns): four 128-column accumulators, one per unit in flight, so
// the epilogues of short units overlap the next units' products.  The product
// is acc (M = 128 queries, N = 128 features, K = 16 keys per step) with A = G
// read from the G^T tile (queries contiguous: MN-major) and B = the K tile
// (features contiguous: MN-major).
#pragma once
#include "sm100.cuh"

namespace ar {

struct DqParams {
  const __nv_bfloat16* q;  // [B, T, H, D]
  const __nv_bfloat16* rcos;  // kRope: rotary tables [>= T, 64], row t = position t
  const __nv_bfloat16* rsin;
  __nv_bfloat16* dq;       // [B, T, H, D]
  int B, T, H;
  int grp;         // query heads per K/V head: k has H / grp heads (1: multi-head)
  int w;           // left window (w >= T means full causal)
  int nq;          // query tiles per head
  int n_units;     // n_bh * nq
  int bh0, n_bh;   // query heads bh0 .. bh0 + n_bh - 1 (b * H + h): the groups of the backward launch's K/V heads
  int nb;          // key tiles in one query tile's band (as in the backward kernel)
  int pairs_head;  // G tiles per head
  float eps, scale;
  int wide;        // dq is 32-byte aligned: rows are written with 256-bit stores
  int wide_q;      // q is 32-byte aligned: query rows are read with 256-bit loads
  unsigned long long wait_ns;  // limit of a device-side wait (kWaitLimitNs unless set otherwise)
};

namespace dqk {
constexpr int kThreads = 224;
constexpr uint32_t kTile = 32768, kHalf = 16384;
constexpr int kGStages = 4, kKStages = 3;
constexpr int kAcc = 4;  // TMEM accumulators (128 columns each)
constexpr uint32_t kG = 0, kK = kGStages * kTile;
enum {
  GFULL = 0, GEMPTY = GFULL + kGStages, KFULL = GEMPTY + kGStages, KEMPTY = KFULL + kKStages,
  ACCFULL = KEMPTY + kKStages, ACCFREE = ACCFULL + kAcc, FINAL = ACCFREE + kAcc, NBAR
};
constexpr uint32_t kBar = kK + kKStages * kTile;
constexpr uint32_t kTmemPtr = kBar + NBAR * 8;
constexpr uint32_t kAbort = kTmemPtr + 4;
constexpr uint32_t kSmemBytes = kAbort + 4 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");

// A unit: query tile qt of one head, with key tiles kt = hi (= qt) down to lo.
struct Unit {
  int hl, bh, b, h, qt, lo, hi;
};

__device__ __forceinline__ int unit_index(int cta, int round, int G) {
  return round * G + ((round & 1) ? (G - 1 - cta) : cta);
}

// Units are (head, query tile), later tiles (longer bands) first.
__device__ __forceinline__ Unit decode(const DqParams& p, int u) {
  Unit U;
  U.hl = u % p.n_bh;
  U.bh = p.bh0 + U.hl;
  U.b = U.bh / p.H;
  U.h = U.bh % p.H;
  U.qt = p.nq - 1 - u / p.n_bh;
  U.lo = max(0, U.qt * 128 - p.w) / 128;
  U.hi = U.qt;
  return U;
}

// Same slot layout as g_pair in the backward kernel.
__device__ __forceinline__ long long g_slot(const DqParams& p, int hl, int qt, int kt) {
  const long long before = qt <= p.nb ? (long long)qt * (qt + 1) / 2
                                      : (long long)p.nb * (p.nb + 1) / 2 + (long long)(qt - p.nb) * p.nb;
  return (long long)hl * p.pairs_head + before + (qt - kt);
}

__device__ __forceinline__ uint32_t bar_addr(uint32_t sbase, int i) { return sbase + kBar + 8u * i; }

template <bool kRope, int kD = 128>
__global__ void __launch_bounds__(kThreads, 1)
    dq_kernel(const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_k, const DqParams p) {
  // Head dimension kD (64 or 128): K tiles are kD / 64 swizzled halves in their
  // 32 KB slots and the accumulator uses kD of its 128 columns.
  static_assert(kD == 64 || kD == 128, "head dimension 64 or 128");
  static_assert(kD == 128 || !kRope, "the RoPE path takes head dimension 128");
  constexpr int kHalves = kD / 64;
  constexpr float kInvD = 1.0f / kD;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kAbort);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int G = gridDim.x, cta = blockIdx.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NBAR; ++i) mbar_init(bar_addr(sbase, i), (i >= ACCFREE && i < ACCFREE + kAcc) ? 128 : 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(sbase + kTmemPtr, 512);
    tmem_relinquish();
  }
  if ((warp == 4 || warp == 6) && lane == 0) {
    prefetch_tmap(&tm_g);
    prefetch_tmap(&tm_k);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *reinterpret_cast<volatile uint32_t*>(smem + kTmemPtr);

  if (warp == 4 || warp == 6) {
    if (lane == 0) {
      // ---------------------------------------------------------- TMA producers: G (warp 4), K (warp 6)
      // Both walk the unit's key tiles newest first.
      const bool is_g = warp == 4;
      const int nst = is_g ? kGStages : kKStages;
      const int full = is_g ? GFULL : KFULL, empty = is_g ? GEMPTY : KEMPTY;
      uint32_t c = 0;
      bool ok = true;
      int last_par[kGStages] = {-1, -1, -1, -1};
      for (int r = 0; ok; ++r) {
        const int u = unit_index(cta, r, G);
        if (u >= p.n_units) break;
        const Unit U = decode(p, u);
        for (int kt = U.hi; kt >= U.lo; --kt, ++c) {
          const int s = c % nst, ph = (c / nst) & 1;
          if (!mbar_wait(bar_addr(sbase, empty + s), ph ^ 1, abort_flag, p.wait_ns)) {
            ok = false;
            break;
          }
          mbar_expect_tx(bar_addr(sbase, full + s), is_g ? kTile : 128u * kD * 2);
          if (is_g) {
            const long long slot = g_slot(p, U.hl, U.qt, kt);
            for (int hf = 0; hf < 2; ++hf)
              tma_load_2d(sbase + kG + s * kTile + hf * kHalf, &tm_g, bar_addr(sbase, full + s), 0,
                          (int)((2 * slot + hf) * 128));
          } else {
            for (int hf = 0; hf < kHalves; ++hf)
              tma_load_4d(sbase + kK + s * kTile + hf * kHalf, &tm_k, bar_addr(sbase, full + s), hf * 64,
                          U.h / p.grp, kt * 128, U.b);
          }
          last_par[s] = ph;
        }
      }
      {
        // Every exit, normal or aborted: the copies still in flight land before
        // the CTA's shared memory goes away (on the normal path they have landed).
        for (int s = 0; s < nst; ++s)
          if (last_par[s] >= 0) mbar_drain(bar_addr(sbase, full + s), last_par[s]);
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      constexpr uint32_t id = idesc_bf16(128, kD, 1, 1);  // A (G) and B (K) both MN-major
      const uint64_t dA = sdesc_sw128(sbase + kG, kHalf, 1024), dB = sdesc_sw128(sbase + kK, kHalf, 1024);
      uint32_t cg = 0, ck = 0;
      int uidx = 0;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int u = unit_index(cta, r, G);
        if (u >= p.n_units) break;
        const Unit U = decode(p, u);
        const int ab = uidx % kAcc;
        if (uidx >= kAcc && !mbar_wait(bar_addr(sbase, ACCFREE + ab), (uidx / kAcc - 1) & 1, abort_flag, p.wait_ns)) break;
        for (int kt = U.hi; kt >= U.lo; --kt, ++ck, ++cg) {
          const int ks = ck % kKStages, kph = (ck / kKStages) & 1;
          const int gs = cg % kGStages, gph = (cg / kGStages) & 1;
          if (!mbar_wait(bar_addr(sbase, KFULL + ks), kph, abort_flag, p.wait_ns) ||
              !mbar_wait(bar_addr(sbase, GFULL + gs), gph, abort_flag, p.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(tbase + 128 * ab, sdesc_add(dA, gs * kTile + kk * 2048), sdesc_add(dB, ks * kTile + kk * 2048),
                   id, (kt < U.hi || kk > 0) ? 1u : 0u);
          mma_commit(bar_addr(sbase, GEMPTY + gs));
          mma_commit(bar_addr(sbase, KEMPTY + ks));
        }
        if (!ok) break;
        mma_commit(bar_addr(sbase, ACCFULL + ab));
        ++uidx;
      }
      mma_commit(bar_addr(sbase, FINAL));
      mbar_drain(bar_addr(sbase, FINAL), 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int row = threadIdx.x;  // TMEM lane = query row of a tile
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    int uidx = 0;
    bool ok = true;
    for (int r = 0; ok; ++r) {
      const int u = unit_index(cta, r, G);
      if (u >= p.n_units) break;
      const Unit U = decode(p, u);
      const int ab = uidx % kAcc;
      {
        const int i = U.qt * 128 + row;
        const bool iv = i < p.T;
        const size_t orow = (((size_t)U.b * p.T + (iv ? i : 0)) * p.H + U.h) * kD;
        // the whole q row, loaded before the wait for the accumulator so that its
        // latency overlaps the products
        uint4 qv[kD / 8];
        {
          const uint4* qrow = reinterpret_cast<const uint4*>(p.q + orow);
#pragma unroll
          for (int c = 0; c < kD / 8; c += 2) {
            if (iv) {
              ldg32B(qrow + c, qv[c], qv[c + 1], p.wide_q);
            } else {
              qv[c] = make_uint4(0, 0, 0, 0);
              qv[c + 1] = qv[c];
            }
          }
        }
        if (!__all_sync(0xffffffffu, mbar_wait(bar_addr(sbase, ACCFULL + ab), (uidx / kAcc) & 1, abort_flag, p.wait_ns))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tA = tbase + 128 * ab + lane_off;
        // pass 1: (acc . q) and sum q^2
        float ss = 0.f, dot = 0.f;
#pragma unroll
        for (int cc = 0; cc < kD / 32; ++cc) {
          uint32_t x[32];
          tmem_ld32(tA + 32 * cc, x);
          tmem_wait_ld();
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const uint4 v = qv[4 * cc + q4];
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float q0 = bf16lo(w4[e]), q1 = bf16hi(w4[e]);
              ss = fmaf(q0, q0, fmaf(q1, q1, ss));
              dot = fmaf(__uint_as_float(x[8 * q4 + 2 * e]), q0, fmaf(__uint_as_float(x[8 * q4 + 2 * e + 1]), q1, dot));
            }
          }
        }
        const float coef = dot * kInvD / (ss * kInvD + p.eps);
        if constexpr (!kRope) {
          // pass 2: dq = scale (acc - coef q)
#pragma unroll
          for (int cc = 0; cc < kD / 32; ++cc) {
            uint32_t x[32];
            tmem_ld32(tA + 32 * cc, x);
            tmem_wait_ld();
            uint32_t pk[16];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              const uint4 v = qv[4 * cc + q4];
              const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float g0 = p.scale * (__uint_as_float(x[8 * q4 + 2 * e]) - coef * bf16lo(w4[e]));
                const float g1 = p.scale * (__uint_as_float(x[8 * q4 + 2 * e + 1]) - coef * bf16hi(w4[e]));
                pk[4 * q4 + e] = pack_bf16(g0, g1);
              }
            }
            if (iv) {
              stg32B(p.dq + orow + 32 * cc, pk, p.wide);
              stg32B(p.dq + orow + 32 * cc + 16, pk + 8, p.wide);
            }
          }
        } else {
          // pass 2: dq_rot = scale (acc - coef q_rot), then dq = R_i^T dq_rot, for
          // features 16c .. 16c+15 with their partners 64 + 16c ..
          const __nv_bfloat16* cr = p.rcos + (size_t)(iv ? i : 0) * 64;
          const __nv_bfloat16* sr = p.rsin + (size_t)(iv ? i : 0) * 64;
#pragma unroll
          for (int c = 0; c < 4; ++c) {  // unrolled: qv is indexed by c
            uint32_t xl[16], xh[16];
            tmem_ld16(tA + 16 * c, xl);
            tmem_ld16(tA + 64 + 16 * c, xh);
            uint4 cv[2], sv[2];
            if (iv) {
              cv[0] = __ldg(reinterpret_cast<const uint4*>(cr + 16 * c));
              cv[1] = __ldg(reinterpret_cast<const uint4*>(cr + 16 * c + 8));
              sv[0] = __ldg(reinterpret_cast<const uint4*>(sr + 16 * c));
              sv[1] = __ldg(reinterpret_cast<const uint4*>(sr + 16 * c + 8));
            } else {
              cv[0] = cv[1] = sv[0] = sv[1] = make_uint4(0, 0, 0, 0);
            }
            tmem_wait_ld();
            uint32_t pl[8], ph[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const uint32_t q1 = (&qv[2 * c + (e >> 2)].x)[e & 3], q2 = (&qv[8 + 2 * c + (e >> 2)].x)[e & 3];
              const uint32_t cw = (&cv[e >> 2].x)[e & 3], sw = (&sv[e >> 2].x)[e & 3];
              const float d10 = p.scale * (__uint_as_float(xl[2 * e]) - coef * bf16lo(q1));
              const float d11 = p.scale * (__uint_as_float(xl[2 * e + 1]) - coef * bf16hi(q1));
              const float d20 = p.scale * (__uint_as_float(xh[2 * e]) - coef * bf16lo(q2));
              const float d21 = p.scale * (__uint_as_float(xh[2 * e + 1]) - coef * bf16hi(q2));
              const float c0 = bf16lo(cw), c1 = bf16hi(cw), s0 = bf16lo(sw), s1 = bf16hi(sw);
              pl[e] = pack_bf16(fmaf(d10, c0, -(d20 * s0)), fmaf(d11, c1, -(d21 * s1)));
              ph[e] = pack_bf16(fmaf(d10, s0, d20 * c0), fmaf(d11, s1, d21 * c1));
            }
            if (iv) {
              stg32B(p.dq + orow + 16 * c, pl, p.wide);
              stg32B(p.dq + orow + 64 + 16 * c, ph, p.wide);
            }
          }
        }
      }
      if (!ok) break;
      tc_fence_before();
      mbar_arrive(bar_addr(sbase, ACCFREE + ab));
      ++uidx;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

}  // namespace dqk
}  // namespace ar
