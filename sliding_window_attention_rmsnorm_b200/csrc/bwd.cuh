// Fused QK-RMSNorm + band-limited causal attention, backward main kernel, sm_100a.
//
// For one head and one tile of 128 keys j, loops over the query tiles i whose
// band reaches those keys and accumulates (s_ij as in the forward pass):
//   P_ij  = exp(s_ij - lse_i)                      recomputed from the saved lse
//   dV_j += sum_i P_ij dO_i
//   dP_ij = dO_i . v_j,  dS_ij = P_ij (dP_ij - delta_i),  delta_i = dO_i . o_i
//   dkhat_j = scale sum_i dS_ij qhat_i,  dqhat_i = scale sum_j dS_ij khat_j
// The RMSNorm enters as the rank-1 factor rq_i rk_j: the tensor core works on
// raw bf16 q and k, and one bf16 matrix G_ij = dS_ij rq_i rk_j feeds both
// gradient products, dK_acc = G^T Q = rk_j dkhat_j / scale and
// dQ_acc = G K = rq_i dqhat_i / scale, which the epilogues correct per row.
// The key-side RMSNorm backward (dk = rk (dkhat - khat (dkhat.khat)/D)) runs in
// this kernel's epilogue; dqhat is accumulated in fp32 in global memory and
// finished by the dq post-pass.
//
// CTA organisation (persistent, one CTA per SM, 320 threads):
//   warps 0-3  compute warpgroup: one key row per thread; P^T, dS^T, epilogue
//   warps 4-7  dQ warpgroup: one query row per thread; reads dQ from TMEM and
//              adds it to the fp32 accumulator with vector reductions
//   warp 8     TMA producer: K, V per unit; Q, dO per query tile (2 stages)
//   warp 9     MMA issuer
// TMEM: S^T (cols 0-127, P^T overwrites 0-63) | dP^T (128-255, later dQ) | dV | dK.
// Shared memory: K, V, Q[2], dO[2], G^T (all 128x128 bf16, 128-byte swizzled),
// plus the per-query vectors (lse*log2 e, delta, rq) of the current tile.
#pragma once
#include "sm100.cuh"

namespace ar {

struct BwdParams {
  __nv_bfloat16* dk;   // [B, T, H, 128]
  __nv_bfloat16* dv;   // [B, T, H, 128]
  float* dq_acc;       // [B, T, H, 128] fp32 dqhat accumulator (zeroed by the pre-pass)
  const float* lse2;   // [B*H, T_pad] lse * log2(e), 0 on padding
  const float* delta;  // [B*H, T_pad] rowsum(dO * o), 0 on padding
  const float* rq;     // [B*H, T_pad] 1/rms(q_i), 0 on padding
  int B, T, H, T_pad;
  int w;        // left window (w >= T means full causal)
  int nk;       // key tiles per head = ceil(T / 128)
  int n_units;  // B * H * nk
  float eps, scale;
};

namespace bwd {
constexpr int kThreads = 384;
// Launch budget 168 registers x 384 threads; warpgroup 2 (TMA, MMA, 2 idle
// warps) drops to 104 so warpgroups 0-1 can rise to 200: 256*200 + 128*104 = 168*384.
constexpr int kRegsLow = 104, kRegsHigh = 200, kLaunchRegs = 168;
static_assert(256 * kRegsHigh + 128 * kRegsLow <= kLaunchRegs * kThreads, "register split exceeds the launch budget");
constexpr uint32_t kTile = 32768, kHalf = 16384;
constexpr uint32_t kK = 0, kV = kTile, kQ = 2 * kTile, kDO = 4 * kTile, kDS = 6 * kTile, kVec = 7 * kTile;
enum {
  KVFULL = 0, KVEMPTY, QFULL, QEMPTY = QFULL + 2, SFULL = QEMPTY + 2, DSREADY, DSFREE, DQFULL, DQFREE,
  DKDVDONE, ACCFREE, VECFULL, VECEMPTY, FINAL, NBAR
};
constexpr uint32_t kBar = kVec + 3 * 512;
constexpr uint32_t kTmemPtr = kBar + NBAR * 8;
constexpr uint32_t kAbort = kTmemPtr + 4;
constexpr uint32_t kSmemBytes = kAbort + 4 + 1024;

struct Unit {
  int bh, b, h, kt, qlo, N;
};

__device__ __forceinline__ int unit_index(int cta, int round, int G) {
  return round * G + ((round & 1) ? (G - 1 - cta) : cta);
}

// Units are (head, key tile), low key tiles first (they see the most queries).
__device__ __forceinline__ Unit decode(const BwdParams& p, int u) {
  Unit U;
  const int BH = p.B * p.H;
  U.kt = u / BH;
  U.bh = u % BH;
  U.b = U.bh / p.H;
  U.h = U.bh % p.H;
  U.qlo = U.kt;
  const long long last_q = (long long)U.kt * 128 + 127 + p.w;
  const int qhi = (int)min((long long)(p.nk - 1), last_q / 128);
  U.N = qhi - U.qlo + 1;
  return U;
}

__device__ __forceinline__ uint32_t bar_addr(uint32_t sbase, int i) { return sbase + kBar + 8u * i; }

__global__ void __launch_bounds__(kThreads, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
               const BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kAbort);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int G = gridDim.x, cta = blockIdx.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NBAR; ++i) {
      uint32_t cnt = 1;
      if (i == DSREADY || i == DQFREE || i == ACCFREE || i == VECFULL || i == VECEMPTY) cnt = 128;
      if (i == KVEMPTY) cnt = 129;  // the MMA commit + every compute thread after its epilogue
      mbar_init(bar_addr(sbase, i), cnt);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(sbase + kTmemPtr, 512);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_do);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *reinterpret_cast<volatile uint32_t*>(smem + kTmemPtr);

  const float kLog2e = 1.4426950408889634f;

  if (warp >= 8) {
   regs_dec<kRegsLow>();
   if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t qc = 0;
      int uidx = 0;
      bool ok = true;
      int last_kv_par = -1, last_q_par[2] = {-1, -1};
      for (int r = 0; ok; ++r) {
        const int u = unit_index(cta, r, G);
        if (u >= p.n_units) break;
        const Unit U = decode(p, u);
        if (uidx > 0 && !mbar_wait(bar_addr(sbase, KVEMPTY), (uidx - 1) & 1, abort_flag)) break;
        mbar_expect_tx(bar_addr(sbase, KVFULL), 2 * kTile);
        for (int hf = 0; hf < 2; ++hf) {
          tma_load_4d(sbase + kK + hf * kHalf, &tm_k, bar_addr(sbase, KVFULL), hf * 64, U.h, U.kt * 128, U.b);
          tma_load_4d(sbase + kV + hf * kHalf, &tm_v, bar_addr(sbase, KVFULL), hf * 64, U.h, U.kt * 128, U.b);
        }
        last_kv_par = uidx & 1;
        for (int it = 0; it < U.N; ++it, ++qc) {
          const int qt = U.qlo + it;
          const int st = qc & 1, ph = (qc >> 1) & 1;
          if (!mbar_wait(bar_addr(sbase, QEMPTY + st), ph ^ 1, abort_flag)) { ok = false; break; }
          mbar_expect_tx(bar_addr(sbase, QFULL + st), 2 * kTile);
          for (int hf = 0; hf < 2; ++hf) {
            tma_load_4d(sbase + kQ + st * kTile + hf * kHalf, &tm_q, bar_addr(sbase, QFULL + st), hf * 64, U.h,
                        qt * 128, U.b);
            tma_load_4d(sbase + kDO + st * kTile + hf * kHalf, &tm_do, bar_addr(sbase, QFULL + st), hf * 64, U.h,
                        qt * 128, U.b);
          }
          last_q_par[st] = ph;
        }
        ++uidx;
      }
      if (*abort_flag) {
        volatile int never = 0;
        if (last_kv_par >= 0) mbar_wait(bar_addr(sbase, KVFULL), last_kv_par, &never);
        for (int s = 0; s < 2; ++s)
          if (last_q_par[s] >= 0) mbar_wait(bar_addr(sbase, QFULL + s), last_q_par[s], &never);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_kk = idesc_bf16(128, 128, 0, 0);  // both operands K-major
      constexpr uint32_t id_kn = idesc_bf16(128, 128, 0, 1);  // A K-major, B MN-major
      constexpr uint32_t id_nn = idesc_bf16(128, 128, 1, 1);  // both MN-major
      const uint32_t tS = tbase, tDP = tbase + 128, tDV = tbase + 256, tDK = tbase + 384;
      uint32_t qc = 0;
      int uidx = 0;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int u = unit_index(cta, r, G);
        if (u >= p.n_units) break;
        const Unit U = decode(p, u);
        if (!mbar_wait(bar_addr(sbase, KVFULL), uidx & 1, abort_flag)) break;
        for (int it = 0; it < U.N; ++it, ++qc) {
          const int st = qc & 1, ph = (qc >> 1) & 1;
          const uint32_t qa = sbase + kQ + st * kTile, da = sbase + kDO + st * kTile;
          if (!mbar_wait(bar_addr(sbase, QFULL + st), ph, abort_flag)) { ok = false; break; }
          tc_fence_after();
          // S^T = K Q^T
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
            mma_ss(tS, sdesc_sw128(sbase + kK + off, 16, 1024), sdesc_sw128(qa + off, 16, 1024), id_kk, kk > 0);
          }
          // dP^T = V dO^T, once the previous dQ has left TMEM
          if (qc > 0 && !mbar_wait(bar_addr(sbase, DQFREE), (qc - 1) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
            mma_ss(tDP, sdesc_sw128(sbase + kV + off, 16, 1024), sdesc_sw128(da + off, 16, 1024), id_kk, kk > 0);
          }
          mma_commit(bar_addr(sbase, SFULL));
          if (!mbar_wait(bar_addr(sbase, DSREADY), qc & 1, abort_flag)) { ok = false; break; }
          if (it == 0 && uidx > 0 && !mbar_wait(bar_addr(sbase, ACCFREE), (uidx - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // dV += P^T dO   (P^T from TMEM)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tDV, tS + kk * 8, sdesc_sw128(da + kk * 2048, kHalf, 1024), id_kn, (it > 0 || kk > 0) ? 1u : 0u);
          // dK += G^T Q
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
            mma_ss(tDK, sdesc_sw128(sbase + kDS + off, 16, 1024), sdesc_sw128(qa + kk * 2048, kHalf, 1024), id_kn,
                   (it > 0 || kk > 0) ? 1u : 0u);
          }
          // dQ = G K   (into the dP^T columns)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(tDP, sdesc_sw128(sbase + kDS + kk * 2048, kHalf, 1024),
                   sdesc_sw128(sbase + kK + kk * 2048, kHalf, 1024), id_nn, kk > 0);
          mma_commit(bar_addr(sbase, DQFULL));
          mma_commit(bar_addr(sbase, DSFREE));
          mma_commit(bar_addr(sbase, QEMPTY + st));
        }
        if (!ok) break;
        mma_commit(bar_addr(sbase, DKDVDONE));
        mma_commit(bar_addr(sbase, KVEMPTY));
        ++uidx;
      }
      mma_commit(bar_addr(sbase, FINAL));
      volatile int never = 0;
      mbar_wait(bar_addr(sbase, FINAL), 0, &never);
    }
  }
  } else {
   regs_inc<kRegsHigh>();
   if (warp < 4) {
    // ------------------------------------------------------------ compute warpgroup (key rows)
    const int row = threadIdx.x;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const uint32_t tS = tbase + lane_off, tDP = tbase + 128 + lane_off;
    const uint32_t tDV = tbase + 256 + lane_off, tDK = tbase + 384 + lane_off;
    float* vec = reinterpret_cast<float*>(smem + kVec);  // [0..127] lse2, [128..255] delta, [256..383] rq
    uint32_t qc = 0;
    int uidx = 0;
    bool ok = true;
    for (int r = 0; ok; ++r) {
      const int u = unit_index(cta, r, G);
      if (u >= p.n_units) break;
      const Unit U = decode(p, u);
      const int j = U.kt * 128 + row;
      if (!__all_sync(0xffffffffu, mbar_wait(bar_addr(sbase, KVFULL), uidx & 1, abort_flag))) break;
      float rk;
      {
        float ss[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 v = lds128(sbase + kK + hf * kHalf + sw128(row, c));
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float a = bf16lo(w4[e]), b2 = bf16hi(w4[e]);
              ss[e] = fmaf(a, a, ss[e]);
              ss[e] = fmaf(b2, b2, ss[e]);
            }
          }
        rk = rsqrtf((ss[0] + ss[1] + ss[2] + ss[3]) * (1.0f / 128.0f) + p.eps);
      }
      const float Cj = rk * p.scale * kLog2e;
      const size_t vbase = (size_t)U.bh * p.T_pad;
      for (int it = 0; it < U.N; ++it, ++qc) {
        const int qt = U.qlo + it;
        // Per-query vectors of this tile, staged through shared memory: every
        // thread writes one entry once all threads are done with the previous tile.
        const float v_lse2 = p.lse2[vbase + qt * 128 + row];
        const float v_delta = p.delta[vbase + qt * 128 + row];
        const float v_rq = p.rq[vbase + qt * 128 + row];
        if (qc > 0 &&
            !__all_sync(0xffffffffu, mbar_wait(bar_addr(sbase, VECEMPTY), (qc - 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
        vec[row] = v_lse2;
        vec[128 + row] = v_delta;
        vec[256 + row] = v_rq;
        mbar_arrive(bar_addr(sbase, VECFULL));
        if (!__all_sync(0xffffffffu, mbar_wait(bar_addr(sbase, VECFULL), qc & 1, abort_flag))) { ok = false; break; }
        if (!__all_sync(0xffffffffu, mbar_wait(bar_addr(sbase, SFULL), qc & 1, abort_flag))) { ok = false; break; }
        if (qc > 0 &&
            !__all_sync(0xffffffffu, mbar_wait(bar_addr(sbase, DSFREE), (qc - 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const bool masked = (qt == U.kt) || (qt * 128 + 127 - U.kt * 128 > p.w) || (qt * 128 + 127 >= p.T);
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t sv[32], dp[32];
          tmem_ld32(tS + 32 * c, sv);
          tmem_ld32(tDP + 32 * c, dp);
          tmem_wait_ld();
          uint32_t pk[16], gk[16];
#pragma unroll
          for (int e2 = 0; e2 < 16; ++e2) {
            float pp[2], gg[2];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int e = 2 * e2 + h2;
              const int ii = 32 * c + e;
              const float rqi = vec[256 + ii];
              float P = ex2(fmaf(__uint_as_float(sv[e]) * rqi, Cj, -vec[ii]));
              if (masked) {
                const int i = qt * 128 + ii;
                if (i < j || i - j > p.w || i >= p.T) P = 0.f;
              }
              const float dS = P * (__uint_as_float(dp[e]) - vec[128 + ii]);
              pp[h2] = P;
              gg[h2] = dS * rqi * rk;
            }
            pk[e2] = pack_bf16(pp[0], pp[1]);
            gk[e2] = pack_bf16(gg[0], gg[1]);
          }
          tmem_st16(tS + 16 * c, pk);
          // G^T row j, queries 32c..32c+31: region c/2, 16-byte chunks 4*(c&1)..+3
          const uint32_t ga = sbase + kDS + (c >> 1) * kHalf;
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            sts128(ga + sw128(row, 4 * (c & 1) + q4),
                   make_uint4(gk[4 * q4], gk[4 * q4 + 1], gk[4 * q4 + 2], gk[4 * q4 + 3]));
        }
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar_addr(sbase, DSREADY));
        mbar_arrive(bar_addr(sbase, VECEMPTY));
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue: dV, dK (with norm backward)
      if (!__all_sync(0xffffffffu, mbar_wait(bar_addr(sbase, DKDVDONE), uidx & 1, abort_flag))) break;
      tc_fence_after();
      const size_t orow = (((size_t)U.b * p.T + j) * p.H + U.h) * 128;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t a[32];
        tmem_ld32(tDV + 32 * c, a);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) pk[e] = pack_bf16(__uint_as_float(a[2 * e]), __uint_as_float(a[2 * e + 1]));
        if (j < p.T) {
          uint4* dst = reinterpret_cast<uint4*>(p.dv + orow + 32 * c);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
      }
      {
        // dk = scale (acc - rk^2 k (acc . k) / D): first the dot product, then the output,
        // each pass reading 32 accumulator columns at a time.
        float dot[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t a[32];
          tmem_ld32(tDK + 32 * c, a);
          tmem_wait_ld();
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const int cc = 4 * c + q4;  // 16-byte chunk of the k row (8 elements)
            const uint4 v = lds128(sbase + kK + (cc >> 3) * kHalf + sw128(row, cc & 7));
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              dot[e] = fmaf(__uint_as_float(a[8 * q4 + 2 * e]), bf16lo(w4[e]), dot[e]);
              dot[e] = fmaf(__uint_as_float(a[8 * q4 + 2 * e + 1]), bf16hi(w4[e]), dot[e]);
            }
          }
        }
        const float coef = rk * rk * ((dot[0] + dot[1]) + (dot[2] + dot[3])) * (1.0f / 128.0f);
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t a[32];
          tmem_ld32(tDK + 32 * c, a);
          tmem_wait_ld();
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const int cc = 4 * c + q4;
            const uint4 v = lds128(sbase + kK + (cc >> 3) * kHalf + sw128(row, cc & 7));
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
            uint32_t o4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float g0 = p.scale * (__uint_as_float(a[8 * q4 + 2 * e]) - coef * bf16lo(w4[e]));
              const float g1 = p.scale * (__uint_as_float(a[8 * q4 + 2 * e + 1]) - coef * bf16hi(w4[e]));
              o4[e] = pack_bf16(g0, g1);
            }
            if (j < p.T)
              *reinterpret_cast<uint4*>(p.dk + orow + 8 * cc) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
          }
        }
        tc_fence_before();
        mbar_arrive(bar_addr(sbase, ACCFREE));
      }
      mbar_arrive(bar_addr(sbase, KVEMPTY));
      ++uidx;
    }
  } else {
    // ------------------------------------------------------------ dQ warpgroup (query rows)
    const int row = threadIdx.x - 128;
    const uint32_t tDQ = tbase + 128 + ((uint32_t)((warp & 3) * 32) << 16);
    uint32_t qc = 0;
    bool ok = true;
    for (int r = 0; ok; ++r) {
      const int u = unit_index(cta, r, G);
      if (u >= p.n_units) break;
      const Unit U = decode(p, u);
      for (int it = 0; it < U.N; ++it, ++qc) {
        const int i = (U.qlo + it) * 128 + row;
        const float rqi = p.rq[(size_t)U.bh * p.T_pad + (U.qlo + it) * 128 + row];
        if (!__all_sync(0xffffffffu, mbar_wait(bar_addr(sbase, DQFULL), qc & 1, abort_flag))) { ok = false; break; }
        tc_fence_after();
        uint32_t a[128];
        tmem_ld32(tDQ + 0, *reinterpret_cast<uint32_t(*)[32]>(&a[0]));
        tmem_ld32(tDQ + 32, *reinterpret_cast<uint32_t(*)[32]>(&a[32]));
        tmem_ld32(tDQ + 64, *reinterpret_cast<uint32_t(*)[32]>(&a[64]));
        tmem_ld32(tDQ + 96, *reinterpret_cast<uint32_t(*)[32]>(&a[96]));
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(bar_addr(sbase, DQFREE));
        if (i < p.T) {
          const float f = p.scale / rqi;
          float* dst = p.dq_acc + (((size_t)U.b * p.T + i) * p.H + U.h) * 128;
#pragma unroll
          for (int c = 0; c < 32; ++c)
            red_add_v4(dst + 4 * c, __uint_as_float(a[4 * c]) * f, __uint_as_float(a[4 * c + 1]) * f,
                       __uint_as_float(a[4 * c + 2]) * f, __uint_as_float(a[4 * c + 3]) * f);
        }
      }
    }
  }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

}  // namespace bwd
}  // namespace ar
