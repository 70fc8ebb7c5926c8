// Fused QK-RMSNorm + band-limited causal attention, backward main kernel, sm_100a.
//
// For one head and one tile of 128 keys j, loops over the query tiles i whose
// band reaches those keys and accumulates (s_ij as in the forward pass; with
// grouped K/V heads the loop runs over those query tiles of every query head
// of the K/V head's group, so dK and dV sum the group's contributions):
//   P_ij  = exp(s_ij - lse_i)                      recomputed from the saved lse
//   dV_j += sum_i P_ij dO_i
//   dP_ij = dO_i . v_j,  dS_ij = P_ij (dP_ij - delta_i),  delta_i = dO_i . o_i
//   dkhat_j = scale sum_i dS_ij qhat_i,  dqhat_i = scale sum_j dS_ij khat_j
// The RMSNorm enters as the rank-1 factor rq_i rk_j: the tensor core works on
// raw bf16 q and k, and one bf16 matrix G_ij = dS_ij rq_i rk_j feeds both
// gradient products, dK_acc = G^T Q = rk_j dkhat_j / scale here and
// dQ_acc = G K = rq_i dqhat_i / scale in the dq kernel (dq.cuh).  The key-side
// RMSNorm backward (dk = rk (dkhat - khat (dkhat.khat)/D)) runs in this
// kernel's epilogue.  Each 128x128 tile of G^T is written to a global buffer
// (one slot per (query tile, key tile) pair of the band) for the dq kernel,
// so no TMEM columns are spent on dQ and no query tile waits for a dQ read-out.
//
// Each 128-query tile is handled as two 64-query halves a = 0, 1, one per
// compute warpgroup, and the MMAs are software-pipelined so that the tensor
// core computes half a of the next tile while the warpgroups finish this one:
//   grad(0,i) dP_0(i+1) S_0(i+1) | grad(1,i) dP_1(i+1) S_1(i+1) | grad(0,i+1) ...
// with grad(a,i) = dV += P_a^T dO_a, dK += G_a^T Q_a.  S_a(i+1) overwrites the
// columns holding P_a^T(i); the tensor core runs one thread's MMAs in order, so
// the dV product has read them first.
//
// CTA organisation (persistent, one CTA per SM, 512 threads):
//   warps 0-3   compute warpgroup 0: query half 0; one key row per thread
//   warps 4-7   compute warpgroup 1: query half 1
//   warps 8-11  epilogue warpgroup: dK, dV of each key tile
//   warp 12     TMA producer: K, V per unit; Q, dO per query tile (2 stages)
//   warp 13     MMA issuer
//   warp 14     TMA store of each G^T half to the global G buffer;  warp 15 idle
// TMEM (512 columns): S_0 | S_1 (64 each; P_a^T overwrites the first 32) |
// dP_0 | dP_1 (64 each) | dV (128) | dK (128).
// Shared memory: K, V, Q[2], dO[2], G^T (all 128x128 bf16, 128-byte swizzled,
// G^T half a = query columns 64a..64a+63), plus per-half query vectors.
//
// With the RoPE / value-embedding prologue (kPro != 0) the tensor maps and p.k
// point at the rotated q, k and the mixed v that the pre-pass wrote (the same
// bf16 values the forward formed in its tiles), and the epilogue finishes the
// chain rule: dk = R_j^T dk_rot (the transposed rotation of the key's position:
// dk1 = d1 cos - d2 sin, dk2 = d1 sin + d2 cos for the halves d1, d2), and for
// the value embedding v_mix = v + gate ve, gate = 2 sigmoid(g): dv = dv_mix,
// dve = gate dv_mix, dg = (dv_mix . ve) gate (1 - gate / 2).
#pragma once
#include "sm100.cuh"

namespace ar {

struct BwdParams {
  __nv_bfloat16* dk;       // [B, T, Hkv, D]
  __nv_bfloat16* dv;       // [B, T, Hkv, D]
  const __nv_bfloat16* k;  // [B, T, Hkv, D] raw keys, for the dk epilogue
  const float* lse2;       // [B*H, T_pad] lse * log2(e), 0 on padding
  const float* delta;      // [B*H, T_pad] rowsum(dO * o), 0 on padding
  const float* rq;         // [B*H, T_pad] 1/rms(q_i), 0 on padding
  int B, T, H, T_pad;
  int Hkv, grp;  // K/V heads and query heads per K/V head (H = Hkv * grp; grp = 1: multi-head)
  int w;        // left window (w >= T means full causal)
  int nk;       // key tiles per head = ceil(T / 128)
  int n_units;  // n_bh * nk
  int bh0, n_bh;   // K/V heads bh0 .. bh0 + n_bh - 1 (b * Hkv + hk) are processed by this launch
  int nb;          // key tiles in one query tile's band: min(nk, floor((w + 127) / 128) + 1)
  int pairs_head;  // G tiles per head: sum over query tiles of min(qt + 1, nb)
  float eps, scale;
  int wide;    // dk and dv are 32-byte aligned: rows are written with 256-bit stores
  int wide_k;  // k is 32-byte aligned: key rows are read with 256-bit loads
  int wide_ve;  // ve is 32-byte aligned
  unsigned long long wait_ns;  // limit of a device-side wait (kWaitLimitNs unless set otherwise)
  const __nv_bfloat16* rcos;   // kPro & 1: rotary tables [>= T, 64], row t = position t
  const __nv_bfloat16* rsin;
  const __nv_bfloat16* ve;     // kPro & 2: value embedding [B, T, Hkv, 128] and gate logits [B, T, Hkv]
  const __nv_bfloat16* vg;
  __nv_bfloat16* dve;          // kPro & 2: outputs [B, T, Hkv, 128] and [B, T, Hkv]
  float* dg;
};

// Slot of the G tile of (query tile qt, key tile kt) of the launch's query head
// number hl (0 .. grp * n_bh - 1) in the G buffer: query tiles in order, each
// followed by its band's key tiles, newest first.
__device__ __forceinline__ long long g_pair(int hl, int qt, int kt, int nb, int pairs_head) {
  const long long before = qt <= nb ? (long long)qt * (qt + 1) / 2
                                    : (long long)nb * (nb + 1) / 2 + (long long)(qt - nb) * nb;
  return (long long)hl * pairs_head + before + (qt - kt);
}

namespace bwd {
constexpr int kThreads = 512;
// 128 registers per thread for every role (65536 / 512); no register moves.
constexpr int kLaunchRegs = 128;
constexpr uint32_t kTile = 32768, kHalf = 16384;
constexpr uint32_t kK = 0, kV = kTile, kQ = 2 * kTile, kDO = 4 * kTile, kG = 6 * kTile, kVec = 7 * kTile;
enum {
  KVFULL = 0, KVEMPTY, QFULL, QEMPTY = QFULL + 2, SFULL = QEMPTY + 2, DSREADY = SFULL + 2, DSFREE = DSREADY + 2,
  VECFULL = DSFREE + 2, VECEMPTY = VECFULL + 2, DKDVDONE = VECEMPTY + 2, ACCFREE, DOTFREE, FINAL, NBAR
};
constexpr uint32_t kVecHalf = 3 * 64 * 4;  // lse2, delta, rq for 64 queries
// per key row and query half: rk^2 / D * sum_i G_ij S_ij (the dk norm-backward coefficient)
constexpr uint32_t kDot = kVec + 2 * kVecHalf;
constexpr uint32_t kBar = kDot + 2 * 128 * 4;
constexpr uint32_t kTmemPtr = kBar + NBAR * 8;
constexpr uint32_t kAbort = kTmemPtr + 4;
// No alignment slack: dynamic shared memory of a kernel without static shared
// memory starts 1024-byte aligned; the kernel checks (DEV_LAYOUT) otherwise.
constexpr uint32_t kSmemBytes = kAbort + 4;
static_assert(kSmemBytes <= 232448, "shared memory budget");

// A unit: K/V head h (flat bh, local hl) and key tile kt.  Its N = grp * nq
// iterations run the nq band query tiles qlo .. qlo + nq - 1 of each query head
// of the group in turn: iteration it is query head h * grp + it / nq, query
// tile qlo + it % nq.
struct Unit {
  int hl, bh, b, h, kt, qlo, nq, N;
  __device__ int qhead(int it) const { return it / nq; }  // group member
  __device__ int qtile(int it) const { return qlo + it % nq; }
};

__device__ __forceinline__ int unit_index(int cta, int round, int G) {
  return round * G + ((round & 1) ? (G - 1 - cta) : cta);
}

// Units are (head, key tile), low key tiles first (they see the most queries).
__device__ __forceinline__ Unit decode(const BwdParams& p, int u) {
  Unit U;
  U.kt = u / p.n_bh;
  U.hl = u % p.n_bh;
  U.bh = p.bh0 + U.hl;
  U.b = U.bh / p.Hkv;
  U.h = U.bh % p.Hkv;
  U.qlo = U.kt;
  const long long last_q = (long long)U.kt * 128 + 127 + p.w;
  const int qhi = (int)min((long long)(p.nk - 1), last_q / 128);
  U.nq = qhi - U.qlo + 1;
  U.N = p.grp * U.nq;
  return U;
}

__device__ __forceinline__ uint32_t bar_addr(uint32_t sbase, int i) { return sbase + kBar + 8u * i; }

// One 32-query chunk of a key row: P = 2^(S rq_i C_j - lse2_i) (zero outside the
// band when MASKED), G = P (dP - delta_i) rq_i rk_j, both packed to bf16 pairs,
// and (dt0, dt1) += sum G S over the chunk (S: the raw logit q_i . k_j), so that
// k_j . dK_acc_j = sum_i G_ij q_i . k_j is known without reading k again.
// Two queries at a time in packed fp32x2 arithmetic.
// vaddr: shared-memory address of this chunk's -lse2 entries; delta follows at
// +256 bytes and rq at +512 bytes.
template <bool MASKED>
__device__ __forceinline__ void grad_chunk(const uint32_t (&sv)[32], const uint32_t (&dp)[32], uint32_t vaddr,
                                           float Cj, float rk, int c_lo, int c_hi, int cbase, uint32_t (&pk)[16],
                                           uint32_t (&gk)[16], float& dt0, float& dt1) {
#pragma unroll
  for (int e4 = 0; e4 < 8; ++e4) {
    const float4 L = lds_f4(vaddr + 16 * e4);  // -lse2
    const float4 Dl = lds_f4(vaddr + 256 + 16 * e4);
    const float4 R = lds_f4(vaddr + 512 + 16 * e4);
    const float nl[4] = {L.x, L.y, L.z, L.w}, dl[4] = {Dl.x, Dl.y, Dl.z, Dl.w}, rv[4] = {R.x, R.y, R.z, R.w};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int e = 4 * e4 + 2 * h;
      float rc0, rc1, t0, t1, x0, x1, rr0, rr1;
      fmul2(rc0, rc1, rv[2 * h], rv[2 * h + 1], Cj, Cj);  // rq_i C_j
      ffma2(t0, t1, __uint_as_float(sv[e]), __uint_as_float(sv[e + 1]), rc0, rc1, nl[2 * h], nl[2 * h + 1]);
      float p0 = ex2(t0), p1 = ex2(t1);
      if (MASKED) {
        p0 = (cbase + e < c_lo || cbase + e > c_hi) ? 0.f : p0;
        p1 = (cbase + e + 1 < c_lo || cbase + e + 1 > c_hi) ? 0.f : p1;
      }
      fsub2(x0, x1, __uint_as_float(dp[e]), __uint_as_float(dp[e + 1]), dl[2 * h], dl[2 * h + 1]);
      fmul2(rr0, rr1, rv[2 * h], rv[2 * h + 1], rk, rk);  // rq_i rk_j
      fmul2(x0, x1, x0, x1, p0, p1);
      fmul2(x0, x1, x0, x1, rr0, rr1);
      ffma2(dt0, dt1, __uint_as_float(sv[e]), __uint_as_float(sv[e + 1]), x0, x1, dt0, dt1);
      pk[e4 * 2 + h] = pack_bf16(p0, p1);
      gk[e4 * 2 + h] = pack_bf16(x0, x1);
    }
  }
}

template <int kPro, int kD = 128>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
               const __grid_constant__ CUtensorMap tm_g, const BwdParams p) {
  constexpr bool kRope = (kPro & 1) != 0, kVe = (kPro & 2) != 0;
  // Head dimension kD (64 or 128): K, V, Q and dO tiles are kD / 64 swizzled
  // halves of 128 rows x 64 elements in their 32 KB slots; S^T and dP^T take
  // kD / 16 K-steps; dV and dK use kD of their 128 accumulator columns.
  static_assert(kD == 64 || kD == 128, "head dimension 64 or 128");
  static_assert(kD == 128 || kPro == 0, "the RoPE / value-embedding path takes head dimension 128");
  constexpr int kHalves = kD / 64;
  constexpr uint32_t kTileBytes = 128u * kD * 2;
  constexpr float kInvD = 1.0f / kD;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  const uint32_t sbase = smem_u32(smem);
  if (sbase & 1023u) {  // uniform over the CTA: every thread returns before any barrier
    if (threadIdx.x == 0) atomicOr(&g_status, DEV_LAYOUT);
    return;
  }
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kAbort);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int G = gridDim.x, cta = blockIdx.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NBAR; ++i) {
      uint32_t cnt = 1;
      if (i == DSREADY || i == DSREADY + 1 || i == VECFULL || i == VECFULL + 1 || i == VECEMPTY ||
          i == VECEMPTY + 1 || i == ACCFREE || i == DOTFREE)
        cnt = 128;
      if (i == DSFREE || i == DSFREE + 1) cnt = 2;  // the MMA commit + the G^T store's read
      if (i == KVEMPTY) cnt = 1 + 256;  // the MMA commit + every compute thread once rk is read
      mbar_init(bar_addr(sbase, i), cnt);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 13) {
    tmem_alloc(sbase + kTmemPtr, 512);
    tmem_relinquish();
  }
  if (warp == 12 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_do);
    prefetch_tmap(&tm_g);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *reinterpret_cast<volatile uint32_t*>(smem + kTmemPtr);
  const float kLog2e = 1.4426950408889634f;

  if (warp >= 12) {
    if (warp == 12 && lane == 0) {
      // ---------------------------------------------------------- TMA producer
      uint32_t qc = 0;
      int uidx = 0;
      bool ok = true;
      int last_kv_par = -1, last_q_par[2] = {-1, -1};
      for (int r = 0; ok; ++r) {
        const int u = unit_index(cta, r, G);
        if (u >= p.n_units) break;
        const Unit U = decode(p, u);
        if (uidx > 0 && !mbar_wait(bar_addr(sbase, KVEMPTY), (uidx - 1) & 1, abort_flag, p.wait_ns)) break;
        mbar_expect_tx(bar_addr(sbase, KVFULL), 2 * kTileBytes);
        for (int hf = 0; hf < kHalves; ++hf) {
          tma_load_4d(sbase + kK + hf * kHalf, &tm_k, bar_addr(sbase, KVFULL), hf * 64, U.h, U.kt * 128, U.b);
          tma_load_4d(sbase + kV + hf * kHalf, &tm_v, bar_addr(sbase, KVFULL), hf * 64, U.h, U.kt * 128, U.b);
        }
        last_kv_par = uidx & 1;
        for (int it = 0; it < U.N; ++it, ++qc) {
          const int qt = U.qtile(it), hq = U.h * p.grp + U.qhead(it);
          const int st = qc & 1, ph = (qc >> 1) & 1;
          if (!mbar_wait(bar_addr(sbase, QEMPTY + st), ph ^ 1, abort_flag, p.wait_ns)) { ok = false; break; }
          mbar_expect_tx(bar_addr(sbase, QFULL + st), 2 * kTileBytes);
          for (int hf = 0; hf < kHalves; ++hf) {
            tma_load_4d(sbase + kQ + st * kTile + hf * kHalf, &tm_q, bar_addr(sbase, QFULL + st), hf * 64, hq,
                        qt * 128, U.b);
            tma_load_4d(sbase + kDO + st * kTile + hf * kHalf, &tm_do, bar_addr(sbase, QFULL + st), hf * 64, hq,
                        qt * 128, U.b);
          }
          last_q_par[st] = ph;
        }
        ++uidx;
      }
      {
        // Every exit, normal or aborted: the copies still in flight land before
        // the CTA's shared memory goes away (on the normal path they have landed).
        if (last_kv_par >= 0) mbar_drain(bar_addr(sbase, KVFULL), last_kv_par);
        for (int s = 0; s < 2; ++s)
          if (last_q_par[s] >= 0) mbar_drain(bar_addr(sbase, QFULL + s), last_q_par[s]);
      }
    } else if (warp == 14 && lane == 0) {
      // ---------------------------------------------------------- G^T stores
      // Each half of G^T, once its compute warpgroup has written it (DSREADY), is
      // stored to its slot of the global G buffer; the shared-memory half is
      // released (the second DSFREE arrival) once the store has read it.
      uint32_t qc = 0;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int u = unit_index(cta, r, G);
        if (u >= p.n_units) break;
        const Unit U = decode(p, u);
        for (int it = 0; it < U.N && ok; ++it, ++qc) {
          const long long pair = g_pair(U.hl * p.grp + U.qhead(it), U.qtile(it), U.kt, p.nb, p.pairs_head);
          for (int a = 0; a < 2; ++a) {
            if (!mbar_wait(bar_addr(sbase, DSREADY + a), qc & 1, abort_flag, p.wait_ns)) {
              ok = false;
              break;
            }
            tma_store_2d(&tm_g, sbase + kG + a * kHalf, 0, (int)((2 * pair + a) * 128));
            bulk_commit();
            bulk_wait_read();
            mbar_arrive(bar_addr(sbase, DSFREE + a));
          }
        }
      }
      bulk_wait_all();  // every G tile has reached global memory
    } else if (warp == 13 && lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      constexpr uint32_t id_s = idesc_bf16(128, 64, 0, 0);     // S^T, dP^T: both K-major, N = 64 queries
      constexpr uint32_t id_acc = idesc_bf16(128, kD, 0, 1);  // dV, dK: A K-major, B MN-major
      const uint32_t tDV = tbase + 256, tDK = tbase + 384;
      auto issue_s = [&](int a, int st) {  // S_a^T = K Q_a^T
        const uint32_t qa = sbase + kQ + st * kTile + a * 64 * 128;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
          mma_ss(tbase + 64 * a, sdesc_sw128(sbase + kK + off, 16, 1024), sdesc_sw128(qa + off, 16, 1024), id_s,
                 kk > 0);
        }
      };
      auto issue_dp = [&](int a, int st) {  // dP_a^T = V dO_a^T
        const uint32_t da = sbase + kDO + st * kTile + a * 64 * 128;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
          mma_ss(tbase + 128 + 64 * a, sdesc_sw128(sbase + kV + off, 16, 1024), sdesc_sw128(da + off, 16, 1024),
                 id_s, kk > 0);
        }
      };
      auto issue_grad = [&](int a, int st, bool first) {
        const uint32_t qrow = sbase + kQ + st * kTile + a * 64 * 128;
        const uint32_t drow = sbase + kDO + st * kTile + a * 64 * 128;
        const uint32_t ga = sbase + kG + a * kHalf;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // dV += P_a^T dO_a   (P_a^T from TMEM, 16 queries per step)
          mma_ts(tDV, tbase + 64 * a + kk * 8, sdesc_sw128(drow + kk * 2048, kHalf, 1024), id_acc,
                 (first && kk == 0) ? 0u : 1u);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // dK += G_a^T Q_a
          mma_ss(tDK, sdesc_sw128(ga + kk * 32, 16, 1024), sdesc_sw128(qrow + kk * 2048, kHalf, 1024), id_acc,
                 (first && kk == 0) ? 0u : 1u);
      };
      uint32_t qc = 0;
      int uidx = 0;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int u = unit_index(cta, r, G);
        if (u >= p.n_units) break;
        const Unit U = decode(p, u);
        if (!mbar_wait(bar_addr(sbase, KVFULL), uidx & 1, abort_flag, p.wait_ns)) break;
        {  // prologue: S and dP of both halves of the first tile
          const int st = qc & 1, ph = (qc >> 1) & 1;
          if (!mbar_wait(bar_addr(sbase, QFULL + st), ph, abort_flag, p.wait_ns)) break;
#pragma unroll
          for (int a = 0; a < 2; ++a) {
            tc_fence_after();
            issue_s(a, st);
            issue_dp(a, st);
            mma_commit(bar_addr(sbase, SFULL + a));
          }
          if (!ok) break;
          // K and V are read only by the S and dP products: once the last of
          // them is issued, the next unit's tiles may start loading
          if (U.N == 1) mma_commit(bar_addr(sbase, KVEMPTY));
        }
        for (int it = 0; it < U.N && ok; ++it) {
          const uint32_t q = qc + it, q1 = q + 1;
          const int st = q & 1, st1 = q1 & 1, ph1 = (q1 >> 1) & 1;
          const bool has_next = it + 1 < U.N;
#pragma unroll
          for (int a = 0; a < 2; ++a) {
            if (!mbar_wait(bar_addr(sbase, DSREADY + a), q & 1, abort_flag, p.wait_ns)) { ok = false; break; }
            if (it == 0 && a == 0 && uidx > 0 &&
                !mbar_wait(bar_addr(sbase, ACCFREE), (uidx - 1) & 1, abort_flag, p.wait_ns)) { ok = false; break; }
            tc_fence_after();
            issue_grad(a, st, it == 0 && a == 0);
            mma_commit(bar_addr(sbase, DSFREE + a));
            if (a == 1) mma_commit(bar_addr(sbase, QEMPTY + st));
            if (has_next) {
              if (a == 0 && !mbar_wait(bar_addr(sbase, QFULL + st1), ph1, abort_flag, p.wait_ns)) { ok = false; break; }
              tc_fence_after();
              issue_dp(a, st1);
              issue_s(a, st1);
              mma_commit(bar_addr(sbase, SFULL + a));
              if (a == 1 && it + 2 == U.N) mma_commit(bar_addr(sbase, KVEMPTY));
            }
          }
        }
        if (!ok) break;
        mma_commit(bar_addr(sbase, DKDVDONE));
        qc += U.N;
        ++uidx;
      }
      mma_commit(bar_addr(sbase, FINAL));
      mbar_drain(bar_addr(sbase, FINAL), 0);
    }
  } else {
    if (warp < 8) {
      // ---------------------------------------------------------- compute warpgroups (key rows)
      const int a = warp / 4;  // query half
      const int row = threadIdx.x & 127;
      const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
      const uint32_t tS = tbase + 64 * a + lane_off, tDP = tbase + 128 + 64 * a + lane_off;
      // per-half query vectors in shared memory: [0,64) -lse2, [64,128) delta, [128,192) rq (floats)
      const uint32_t vaddr = sbase + kVec + a * kVecHalf;
      const uint32_t ga = sbase + kG + a * kHalf;
      uint32_t qc = 0;
      int uidx = 0;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int u = unit_index(cta, r, G);
        if (u >= p.n_units) break;
        const Unit U = decode(p, u);
        const int j = U.kt * 128 + row;
        if (!__all_sync(0xffffffffu, mbar_wait(bar_addr(sbase, KVFULL), uidx & 1, abort_flag, p.wait_ns))) break;
        float rk;
        {
          float ss[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int hf = 0; hf < kHalves; ++hf)
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const uint4 v = lds128(sbase + kK + hf * kHalf + sw128(row, c));
              const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float x0 = bf16lo(w4[e]), x1 = bf16hi(w4[e]);
                ss[e] = fmaf(x0, x0, ss[e]);
                ss[e] = fmaf(x1, x1, ss[e]);
              }
            }
          rk = rsqrtf((ss[0] + ss[1] + ss[2] + ss[3]) * kInvD + p.eps);
        }
        mbar_arrive(bar_addr(sbase, KVEMPTY));  // done reading K from shared memory
        const float Cj = rk * p.scale * kLog2e;
        float dt0 = 0.f, dt1 = 0.f;
        for (int it = 0; it < U.N; ++it, ++qc) {
          const int qt = U.qtile(it);
          const size_t vbase = ((size_t)U.b * p.H + U.h * p.grp + U.qhead(it)) * p.T_pad;
          const int i0 = qt * 128 + 64 * a;  // first query of this half
          // per-query vectors of this half, staged through shared memory
          const int vsel = row >> 6, vq = row & 63;
          const float v0 = vsel == 0 ? p.lse2[vbase + i0 + vq] : p.rq[vbase + i0 + vq];
          const float v1 = vsel == 0 ? p.delta[vbase + i0 + vq] : 0.f;
          if (qc > 0 &&
              !__all_sync(0xffffffffu, mbar_wait(bar_addr(sbase, VECEMPTY + a), (qc - 1) & 1, abort_flag, p.wait_ns))) {
            ok = false;
            break;
          }
          if (vsel == 0) {
            sts_f32(vaddr + 4 * vq, -v0);  // grad_chunk adds -lse2
            sts_f32(vaddr + 256 + 4 * vq, v1);
          } else {
            sts_f32(vaddr + 512 + 4 * vq, v0);
          }
          mbar_arrive(bar_addr(sbase, VECFULL + a));
          if (!__all_sync(0xffffffffu, mbar_wait(bar_addr(sbase, VECFULL + a), qc & 1, abort_flag, p.wait_ns))) {
            ok = false;
            break;
          }
          if (!__all_sync(0xffffffffu, mbar_wait(bar_addr(sbase, SFULL + a), qc & 1, abort_flag, p.wait_ns))) {
            ok = false;
            break;
          }
          if (qc > 0 &&
              !__all_sync(0xffffffffu, mbar_wait(bar_addr(sbase, DSFREE + a), (qc - 1) & 1, abort_flag, p.wait_ns))) {
            ok = false;
            break;
          }
          tc_fence_after();
          // queries c (0..63) of this half visible to key j: c_lo <= c <= c_hi
          const int c_lo = j - i0;
          const int c_hi = min(j + p.w, p.T - 1) - i0;
          const bool masked = (c_lo > 0) || (c_hi < 63);
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            uint32_t sv[32], dp[32];
            tmem_ld32(tS + 32 * c, sv);
            tmem_ld32(tDP + 32 * c, dp);
            tmem_wait_ld();
            uint32_t pk[16], gk[16];
            if (masked)
              grad_chunk<true>(sv, dp, vaddr + 128 * c, Cj, rk, c_lo, c_hi, 32 * c, pk, gk, dt0, dt1);
            else
              grad_chunk<false>(sv, dp, vaddr + 128 * c, Cj, rk, c_lo, c_hi, 32 * c, pk, gk, dt0, dt1);
            tmem_st16(tS + 16 * c, pk);
            // G^T row j, queries 32c..32c+31 of this half: 16-byte chunks 4c..4c+3
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
              sts128(ga + sw128(row, 4 * c + q4),
                     make_uint4(gk[4 * q4], gk[4 * q4 + 1], gk[4 * q4 + 2], gk[4 * q4 + 3]));
          }
          if (it + 1 == U.N) {
            // this half's share of the dk coefficient, published before the last
            // DSREADY (so the epilogue's wait for the final products covers it) and
            // once the epilogue has taken the previous unit's (DOTFREE)
            if (uidx > 0 &&
                !__all_sync(0xffffffffu, mbar_wait(bar_addr(sbase, DOTFREE), (uidx - 1) & 1, abort_flag, p.wait_ns))) {
              ok = false;
              break;
            }
            sts_f32(sbase + kDot + 4 * (128 * a + row), (dt0 + dt1) * rk * rk * kInvD);
          }
          tmem_wait_st();
          fence_proxy_async_smem();
          tc_fence_before();
          mbar_arrive(bar_addr(sbase, DSREADY + a));
          mbar_arrive(bar_addr(sbase, VECEMPTY + a));
        }
        if (!ok) break;
        ++uidx;
      }
    } else {
      // ---------------------------------------------------------- dK, dV epilogue warpgroup
      const int row = threadIdx.x - 256;  // TMEM lane: key row
      const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
      const uint32_t tDV = tbase + 256 + lane_off, tDK = tbase + 384 + lane_off;
      int uidx = 0;
      for (int r = 0;; ++r) {
        const int u = unit_index(cta, r, G);
        if (u >= p.n_units) break;
        const Unit U = decode(p, u);
        // ------------------------------------------------------------ dK, dV epilogue
        const int j = U.kt * 128 + row;
        const size_t orow = (((size_t)U.b * p.T + (j < p.T ? j : 0)) * p.Hkv + U.h) * kD;
        const bool jv = j < p.T;
        // dk = scale (acc - coef k), coef = rk^2 (acc . k) / D, with acc . k summed by
        // the compute warpgroups as sum_i G_ij S_ij; the raw key row is loaded into
        // registers before the wait, so its latency is hidden by the unit's products
        {
          uint4 kv[kD / 8];
          {
            const uint4* krow = reinterpret_cast<const uint4*>(p.k + orow);
#pragma unroll
            for (int c = 0; c < kD / 8; c += 2) {
              if (jv) {
                ldg32B(krow + c, kv[c], kv[c + 1], p.wide_k);
              } else {
                kv[c] = make_uint4(0, 0, 0, 0);
                kv[c + 1] = kv[c];
              }
            }
          }
          if (!__all_sync(0xffffffffu, mbar_wait(bar_addr(sbase, DKDVDONE), uidx & 1, abort_flag, p.wait_ns))) break;
          tc_fence_after();
          const float coef = lds_f32(sbase + kDot + 4 * row) + lds_f32(sbase + kDot + 4 * (128 + row));
          mbar_arrive(bar_addr(sbase, DOTFREE));
          if constexpr (!kRope) {
#pragma unroll
            for (int c = 0; c < kD / 32; ++c) {
              uint32_t x[32];
              tmem_ld32(tDK + 32 * c, x);
              tmem_wait_ld();
              uint32_t pk[16];
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4) {
                const uint4 v = kv[4 * c + q4];
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const float g0 = p.scale * (__uint_as_float(x[8 * q4 + 2 * e]) - coef * bf16lo(w4[e]));
                  const float g1 = p.scale * (__uint_as_float(x[8 * q4 + 2 * e + 1]) - coef * bf16hi(w4[e]));
                  pk[4 * q4 + e] = pack_bf16(g0, g1);
                }
              }
              if (jv) {
                stg32B(p.dk + orow + 32 * c, pk, p.wide);
                stg32B(p.dk + orow + 32 * c + 16, pk + 8, p.wide);
              }
            }
          } else {
            // dk_rot = scale (acc - coef k_rot) (k_rot: the rotated key row in kv),
            // then dk = R_j^T dk_rot: features 16c .. 16c+15 with their partners
            // 64 + 16c .., the table entries read as needed (the tables stay in L2)
            const __nv_bfloat16* cr = p.rcos + (size_t)(jv ? j : 0) * 64;
            const __nv_bfloat16* sr = p.rsin + (size_t)(jv ? j : 0) * 64;
#pragma unroll
            for (int c = 0; c < 4; ++c) {  // unrolled: kv is indexed by c
              uint32_t xl[16], xh[16];
              tmem_ld16(tDK + 16 * c, xl);
              tmem_ld16(tDK + 64 + 16 * c, xh);
              uint4 cc[2], sc[2];
              if (jv) {
                cc[0] = __ldg(reinterpret_cast<const uint4*>(cr + 16 * c));
                cc[1] = __ldg(reinterpret_cast<const uint4*>(cr + 16 * c + 8));
                sc[0] = __ldg(reinterpret_cast<const uint4*>(sr + 16 * c));
                sc[1] = __ldg(reinterpret_cast<const uint4*>(sr + 16 * c + 8));
              } else {
                cc[0] = cc[1] = sc[0] = sc[1] = make_uint4(0, 0, 0, 0);
              }
              tmem_wait_ld();
              uint32_t pl[8], ph[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const uint32_t kw1 = (&kv[2 * c + (e >> 2)].x)[e & 3], kw2 = (&kv[8 + 2 * c + (e >> 2)].x)[e & 3];
                const uint32_t cw = (&cc[e >> 2].x)[e & 3], sw = (&sc[e >> 2].x)[e & 3];
                const float d10 = p.scale * (__uint_as_float(xl[2 * e]) - coef * bf16lo(kw1));
                const float d11 = p.scale * (__uint_as_float(xl[2 * e + 1]) - coef * bf16hi(kw1));
                const float d20 = p.scale * (__uint_as_float(xh[2 * e]) - coef * bf16lo(kw2));
                const float d21 = p.scale * (__uint_as_float(xh[2 * e + 1]) - coef * bf16hi(kw2));
                const float c0 = bf16lo(cw), c1 = bf16hi(cw), s0 = bf16lo(sw), s1 = bf16hi(sw);
                pl[e] = pack_bf16(fmaf(d10, c0, -(d20 * s0)), fmaf(d11, c1, -(d21 * s1)));
                ph[e] = pack_bf16(fmaf(d10, s0, d20 * c0), fmaf(d11, s1, d21 * c1));
              }
              if (jv) {
                stg32B(p.dk + orow + 16 * c, pl, p.wide);
                stg32B(p.dk + orow + 64 + 16 * c, ph, p.wide);
              }
            }
          }
        }
        if constexpr (!kVe) {
#pragma unroll 1
          for (int c = 0; c < kD / 32; ++c) {
            uint32_t x[32];
            tmem_ld32(tDV + 32 * c, x);
            tmem_wait_ld();
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) pk[e] = pack_bf16(__uint_as_float(x[2 * e]), __uint_as_float(x[2 * e + 1]));
            if (jv) {
              stg32B(p.dv + orow + 32 * c, pk, p.wide);
              stg32B(p.dv + orow + 32 * c + 16, pk + 8, p.wide);
            }
          }
        } else {
          // dv = dv_mix, dve = gate dv_mix, dg = (dv_mix . ve) gate (1 - gate / 2)
          const size_t tok = ((size_t)U.b * p.T + (jv ? j : 0)) * p.Hkv + U.h;
          const float gate = jv ? ve_gate(p.vg[tok]) : 0.f;
          float dot0 = 0.f, dot1 = 0.f;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t x[32];
            tmem_ld32(tDV + 32 * c, x);
            uint4 ev[4];
            if (jv) {
              ldg32B(p.ve + orow + 32 * c, ev[0], ev[1], p.wide_ve);
              ldg32B(p.ve + orow + 32 * c + 16, ev[2], ev[3], p.wide_ve);
            } else {
              ev[0] = ev[1] = ev[2] = ev[3] = make_uint4(0, 0, 0, 0);
            }
            tmem_wait_ld();
            uint32_t pk[16], pe[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float x0 = __uint_as_float(x[2 * e]), x1 = __uint_as_float(x[2 * e + 1]);
              const uint32_t ew = (&ev[e >> 2].x)[e & 3];
              pk[e] = pack_bf16(x0, x1);
              pe[e] = pack_bf16(gate * x0, gate * x1);
              dot0 = fmaf(x0, bf16lo(ew), dot0);
              dot1 = fmaf(x1, bf16hi(ew), dot1);
            }
            if (jv) {
              stg32B(p.dv + orow + 32 * c, pk, p.wide);
              stg32B(p.dv + orow + 32 * c + 16, pk + 8, p.wide);
              stg32B(p.dve + orow + 32 * c, pe, p.wide);
              stg32B(p.dve + orow + 32 * c + 16, pe + 8, p.wide);
            }
          }
          if (jv) p.dg[tok] = (dot0 + dot1) * gate * (1.0f - 0.5f * gate);
        }
        tc_fence_before();
        mbar_arrive(bar_addr(sbase, ACCFREE));
        ++uidx;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

}  // namespace bwd
}  // namespace ar
