// Fused QK-RMSNorm + band-limited causal attention, forward, for sm_100a.
//
// Computes, per head, o_i = sum_j softmax_j(s_ij) v_j and lse_i over the keys
// visible to query i (0 <= i - j <= w), with s_ij = scale * qhat_i . khat_j and
// qhat = q / rms(q), khat = k / rms(k) (parameter-free RMSNorm).  Sources:
// "autoresearch" README (gitee), section 7.3 (norm(q), norm(k) before the
// attention product) and sections 5.2.1-5.2.2 (FlashAttention-3 call with
// window_size = (w, 0), "SSSL" window pattern).
//
// The norm is folded into the logits as a rank-1 scale: the tensor core
// multiplies the raw bf16 q and k, and the softmax warps apply
// rq_i * (rk_j * scale * log2 e), where rq_i comes from the Q tile in shared
// memory and the per-key factor (`ck`) from the K tile, computed by the
// key-factor warps below.  q and k are never rounded after normalisation.
//
// CTA organisation (persistent, one CTA per SM, 512 threads):
//   warps 0-3  softmax warpgroup 0: query tile 0 (rows r0..r0+127), one row per thread
//   warps 4-7  softmax warpgroup 1: query tile 1 (rows r0+128..r0+255)
//   warp 8     TMA producer: Q tiles, K tiles (3 stages), V tiles (2 stages)
//   warp 9     MMA issuer: S_k = Q_k K^T into TMEM, O_k += P_k V with P_k read from TMEM
//   warps 10-11 idle
//   warps 12-15 key factors: ck_j = rk_j * scale * log2(e) of each K tile, one key
//              row per thread, from the tile in shared memory into a 4-slot ring
//              read by the softmax.  One warp sits on each SM sub-partition, so
//              this work takes issue slots evenly from the softmax warps beside it
//              (kCkGlobal: read instead from a [B*H, T_pad] vector in global memory,
//              loaded with the V tile into a slot per V stage; warps 12-15 then idle)
// TMEM (512 columns): S0 | S1 | O0 | O1, 128 fp32 columns each; P_k (bf16
// pairs) overwrites the first 64 columns of S_k.  The MMA issue order
// S0 S1 | PV0 S0' PV1 S1' | ... lets one warpgroup's softmax run while the
// tensor core works for the other.
// Only key tiles that intersect the band of a query tile are visited, in
// descending order from the diagonal tile.
//
// Softmax offset.  The norm bounds every logit: |qhat . khat| <= D, because
// |qhat|^2 = sum q^2 / (mean q^2 + eps) <= D, and likewise for khat; so
// |s_ij log2 e| <= scale D log2 e =: bound.  When bound <= kFixedBoundMax (the
// default scale 1/sqrt(128) gives 16.3), p_ij = 2^(s_ij log2 e - bound) lies in
// [2^-2 bound, 1] for every row, with no underflow in fp32 or bf16, and the
// kernel uses that fixed offset instead of a running row max: one streaming
// pass per tile, no max reduction and no rescaling of O.  Otherwise
// (kFixed = false) it keeps the running max, raised lazily only when it grows
// by more than 2^8.  With the fixed offset no exponential is exactly 1, so O is
// normalised by the sum of the bf16-rounded p that the P V product used (lse
// still takes the unrounded sum); o is then a convex combination of v rows
// with weights that sum to 1 up to fp32 rounding.
// The epilogue writes each thread's normalised O row straight from registers
// to global memory, so a unit's Q buffers are free as soon as its last S
// product has run: the next unit's Q tiles load under the last tile's softmax
// and the epilogue.
//
// RoPE on Q in the tile (kRopeQ): the rotary position embedding of the
// "autoresearch" README (gitee), section 7.4 (the halves x1 = x[:64],
// x2 = x[64:] of each row at position t become x1 cos_t + x2 sin_t and
// -x1 sin_t + x2 cos_t, with bf16 tables) is applied to the unit's two Q tiles
// in shared memory by the key-factor warps when they land, and the MMA warp and
// the softmax warpgroups wait for the rotated tiles (QREADY) instead of the TMA
// arrival.  A Q tile is loaded once per unit, so this costs one pass over q.
// K and V tiles are re-read by every unit whose band covers them (about 4.5
// times per layer at T = 2048, window 1024), so the rotated k and the mixed v
// (section 5.2.3) come from one pre-pass instead (aux.cuh): rotating them in
// each tile was measured at 121 against 54 us per layer, bound by the latency
// of the table and value-embedding loads.
#pragma once
#include <type_traits>

#include "sm100.cuh"

namespace ar {

struct FwdParams {
  __nv_bfloat16* o;  // [B, T, H, D]
  const __nv_bfloat16* rcos;  // kRopeQ: rotary tables [>= T, 64] bf16, row t = position t
  const __nv_bfloat16* rsin;
  float* lse;        // [B, H, T], or NULL: not stored (forward-only use)
  const float* ck;   // kCkGlobal only: [B*Hkv, T_pad] rk_j * scale * log2(e), 0 on padding
  int B, T, H, T_pad;
  int grp;           // query heads per K/V head: k, v have H / grp heads (1: multi-head)
  int w;             // left window (w >= T means full causal)
  int nqp;           // query-tile pairs per head = ceil(T / 256)
  int n_units;       // B * H * nqp
  float eps;
  float bound;       // scale * D * log2(e): the largest |logit| in log2 units
  float cscale;      // scale * log2(e)
  int wide;          // o is 32-byte aligned: rows are written with 256-bit stores
  unsigned long long wait_ns;  // limit of a device-side wait (kWaitLimitNs unless set otherwise)
};

namespace fwd {
constexpr int kThreads = 512;
// Launch budget 128 registers x 512 threads; warpgroup 2 (TMA, MMA, 2 idle
// warps) drops to 104 and warpgroup 3 (key factors) to 40 so warpgroups 0-1 can
// rise to 184: 256*184 + 128*104 + 128*40 = 128*512.  (The running-max softmax
// spills a few registers at 184; the fixed-offset one does not.)
constexpr int kRegsLow = 104, kRegsCk = 40, kRegsHigh = 184, kLaunchRegs = 128;
static_assert(256 * kRegsHigh + 128 * kRegsLow + 128 * kRegsCk <= kLaunchRegs * kThreads,
              "register split exceeds the launch budget");
// With the rotation of Q the key-factor warps take 56 registers; the softmax
// warpgroups give up the difference.
constexpr int kRegsLowPro = 104, kRegsCkPro = 56, kRegsHighPro = 176;
static_assert(256 * kRegsHighPro + 128 * kRegsLowPro + 128 * kRegsCkPro <= kLaunchRegs * kThreads,
              "register split exceeds the launch budget");
constexpr uint32_t kTile = 32768, kHalf = 16384;
// Stage counts: a K tile is needed first (S = Q K^T) and its loads, which take
// ~5000 cycles under load, were what held the pipeline with two stages; V tiles
// are needed one softmax later and two stages keep them ahead.
constexpr int kKStages = 3, kVStages = 2;
// Key-factor ring: the slot of tile n is free once tile n's K load has been
// issued, because that load waited for the MMAs of tile n - kKStages, which were
// issued after both softmax warpgroups finished tile n - kKStages - 1.
constexpr int kCkSlots = kKStages + 1;
constexpr uint32_t kQ = 0, kK = 2 * kTile, kV = kK + kKStages * kTile, kCK = kV + kVStages * kTile;
// Largest logit bound (log2 units) for which the fixed softmax offset is used:
// p >= 2^-64 stays a normal number in fp32 and bf16.
constexpr float kFixedBoundMax = 32.0f;
enum {
  QFULL = 0, QEMPTY, KFULL, KEMPTY = KFULL + kKStages, VFULL = KEMPTY + kKStages, VEMPTY = VFULL + kVStages,
  SFULL = VEMPTY + kVStages, PFULL = SFULL + 2, ODONE = PFULL + 2, OFREE = ODONE + 2,
  CKFULL = OFREE + 2, FINAL = CKFULL + kCkSlots, QREADY /* kRopeQ only */, NBAR
};
constexpr int kCkThreads = 128;  // warps 12-15
constexpr uint32_t kBar = kCK + kCkSlots * 512;
constexpr uint32_t kTmemPtr = kBar + NBAR * 8;
constexpr uint32_t kAbort = kTmemPtr + 4;
// No alignment slack: the dynamic shared memory of a kernel without static
// shared memory starts 1024-byte aligned; the kernel checks and refuses to run
// (DEV_LAYOUT) otherwise.
constexpr uint32_t kSmemBytes = kAbort + 4;
static_assert(kSmemBytes <= 232448, "shared memory budget");

struct Unit {
  int bh, b, h;
  int hk;  // K/V head read by query head h
  int r0[2];
  bool valid[2];
  int lo[2], hi[2];
  int hi_u, N;
  __device__ bool in(int k, int n) const { return valid[k] && n >= lo[k] && n <= hi[k]; }
};

// Units are (head, query-tile pair); heavier pairs (later rows) first, dealt to
// CTAs in snake order so each CTA's total work is balanced.
__device__ __forceinline__ int unit_index(int cta, int round, int G) {
  return round * G + ((round & 1) ? (G - 1 - cta) : cta);
}

__device__ __forceinline__ Unit decode(const FwdParams& p, int u) {
  Unit U;
  const int BH = p.B * p.H;
  const int qp = p.nqp - 1 - u / BH;
  U.bh = u % BH;
  U.b = U.bh / p.H;
  U.h = U.bh % p.H;
  U.hk = U.h / p.grp;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    U.r0[k] = qp * 256 + 128 * k;
    U.valid[k] = U.r0[k] < p.T;
    const int r1 = min(U.r0[k] + 127, p.T - 1);
    U.lo[k] = max(0, U.r0[k] - p.w) / 128;
    U.hi[k] = r1 / 128;
  }
  U.hi_u = U.valid[1] ? U.hi[1] : U.hi[0];
  U.N = U.hi_u - U.lo[0] + 1;
  return U;
}

__device__ __forceinline__ uint32_t bar_addr(uint32_t sbase, int i) { return sbase + kBar + 8u * i; }

// Rotates, in place, row `row` of a 128-byte-swizzled 128x128 bf16 tile at
// shared address `tile` (features 0-63 in the first 16 KB half, 64-127 in the
// second) by the table rows c, s of its position; the new values are rounded
// to bf16 once.  kRopeChunks 16-byte chunks of each half per pass, their table
// entries loaded first.
constexpr int kRopeChunks = 4;
__device__ __forceinline__ void rope_row(uint32_t tile, int row, const __nv_bfloat16* c, const __nv_bfloat16* s) {
#pragma unroll
  for (int pass = 0; pass < 8 / kRopeChunks; ++pass) {
    uint4 cc[kRopeChunks], sc[kRopeChunks];
#pragma unroll
    for (int i = 0; i < kRopeChunks; ++i) {
      cc[i] = __ldg(reinterpret_cast<const uint4*>(c) + kRopeChunks * pass + i);
      sc[i] = __ldg(reinterpret_cast<const uint4*>(s) + kRopeChunks * pass + i);
    }
#pragma unroll
    for (int i = 0; i < kRopeChunks; ++i) {
      const uint32_t a1 = tile + sw128(row, kRopeChunks * pass + i), a2 = a1 + kHalf;
      const uint4 x1 = lds128(a1), x2 = lds128(a2);
      uint4 y1, y2;
      rope_word(x1.x, x2.x, cc[i].x, sc[i].x, y1.x, y2.x);
      rope_word(x1.y, x2.y, cc[i].y, sc[i].y, y1.y, y2.y);
      rope_word(x1.z, x2.z, cc[i].z, sc[i].z, y1.z, y2.z);
      rope_word(x1.w, x2.w, cc[i].w, sc[i].w, y1.w, y2.w);
      sts128(a1, y1);
      sts128(a2, y2);
    }
  }
}

template <bool kFixed, bool kCkGlobal, bool kRopeQ = false, int kD = 128>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  constexpr bool kRope = kRopeQ;
  static_assert(!(kRopeQ && kCkGlobal), "the rotation of Q runs on the key-factor warps");
  // Head dimension kD (64 or 128): a Q, K or V tile is kD / 64 swizzled halves of
  // 128 rows x 64 elements in its 32 KB slot; QK^T takes kD / 16 K-steps and P V
  // writes kD accumulator columns.
  static_assert(kD == 64 || kD == 128, "head dimension 64 or 128");
  static_assert(!(kD != 128 && (kRopeQ || kCkGlobal)), "RoPE and the no-alloc forward take head dimension 128");
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
      if (i == PFULL || i == PFULL + 1 || i == OFREE || i == OFREE + 1) cnt = 128;
      if (!kCkGlobal && i >= KEMPTY && i < KEMPTY + kKStages) cnt = 1 + kCkThreads;  // MMA commit + key-factor warps
      if (i >= CKFULL && i < CKFULL + kCkSlots) cnt = kCkThreads;
      if (i == QREADY) cnt = kCkThreads;  // the key-factor warps, once the unit's Q tiles are rotated
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
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *reinterpret_cast<volatile uint32_t*>(smem + kTmemPtr);

  if (warp >= 12) {
    regs_dec<kRope ? kRegsCkPro : kRegsCk>();
    if (!kCkGlobal) {
      // ---------------------------------------------------------- key factors (and Q rotation)
      // Tile kv's factors go to ring slot kv % kCkSlots (free: see kCkSlots).
      const int row = threadIdx.x - 384;  // key row within the tile
      uint32_t kv = 0;
      int uidx = 0;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int u = unit_index(cta, r, G);
        if (u >= p.n_units) break;
        const Unit U = decode(p, u);
        if constexpr (kRope) {
          // the unit's Q tiles: row `row` of each, at its position
          if (!__all_sync(0xffffffffu, mbar_wait(bar_addr(sbase, QFULL), uidx & 1, abort_flag, p.wait_ns))) break;
#pragma unroll 1
          for (int k = 0; k < 2; ++k) {
            const int i = U.r0[k] + row;
            if (U.valid[k] && i < p.T)
              rope_row(sbase + kQ + k * kTile, row, p.rcos + (size_t)i * 64, p.rsin + (size_t)i * 64);
          }
          fence_proxy_async_smem();
          mbar_arrive(bar_addr(sbase, QREADY));
        }
        for (int it = 0; it < U.N; ++it, ++kv) {
          const int n = U.hi_u - it;
          const int st = kv % kKStages, ph = (kv / kKStages) & 1;
          if (!__all_sync(0xffffffffu, mbar_wait(bar_addr(sbase, KFULL + st), ph, abort_flag, p.wait_ns))) {
            ok = false;
            break;
          }
          const uint32_t kt = sbase + kK + st * kTile;
          const int j = n * 128 + row;  // key position
          float s0 = 0.f, s1 = 0.f;
#pragma unroll 1
          for (int c = 0; c < kD / 8; ++c) {  // 16-byte chunk c of the row
            const uint4 x = lds128(kt + (c >> 3) * kHalf + sw128(row, c & 7));
            fma_sq_bf16x2_f32(s0, s1, x.x);
            fma_sq_bf16x2_f32(s0, s1, x.y);
            fma_sq_bf16x2_f32(s0, s1, x.z);
            fma_sq_bf16x2_f32(s0, s1, x.w);
          }
          const float ck = (j < p.T) ? rsqrtf((s0 + s1) * kInvD + p.eps) * p.cscale : 0.f;
          sts_f32(sbase + kCK + (kv % kCkSlots) * 512 + 4 * row, ck);
          mbar_arrive(bar_addr(sbase, KEMPTY + st));  // done with the K tile
          mbar_arrive(bar_addr(sbase, CKFULL + kv % kCkSlots));
        }
        ++uidx;
      }
    }
  } else if (warp >= 8) {
    regs_dec<kRope ? kRegsLowPro : kRegsLow>();
    if (warp == 8 && lane == 0) {
      // ---------------------------------------------------------- TMA producer
      uint32_t kv = 0;
      int uidx = 0;
      bool ok = true;
      int last_k_par[kKStages] = {-1, -1, -1}, last_v_par[kVStages] = {-1, -1}, last_q_par = -1;
      for (int r = 0; ok; ++r) {
        const int u = unit_index(cta, r, G);
        if (u >= p.n_units) break;
        const Unit U = decode(p, u);
        if (uidx > 0 && !mbar_wait(bar_addr(sbase, QEMPTY), (uidx - 1) & 1, abort_flag, p.wait_ns)) break;
        mbar_expect_tx(bar_addr(sbase, QFULL), kTileBytes * (U.valid[1] ? 2 : 1));
        for (int k = 0; k < 2; ++k)
          if (U.valid[k])
            for (int hf = 0; hf < kHalves; ++hf)
              tma_load_4d(sbase + kQ + k * kTile + hf * kHalf, &tm_q, bar_addr(sbase, QFULL), hf * 64, U.h,
                          U.r0[k], U.b);
        last_q_par = uidx & 1;
        for (int it = 0; it < U.N; ++it, ++kv) {
          const int n = U.hi_u - it;
          const int st = kv % kKStages, ph = (kv / kKStages) & 1;
          if (!mbar_wait(bar_addr(sbase, KEMPTY + st), ph ^ 1, abort_flag, p.wait_ns)) { ok = false; break; }
          mbar_expect_tx(bar_addr(sbase, KFULL + st), kTileBytes);
          for (int hf = 0; hf < kHalves; ++hf)
            tma_load_4d(sbase + kK + st * kTile + hf * kHalf, &tm_k, bar_addr(sbase, KFULL + st), hf * 64, U.hk,
                        n * 128, U.b);
          last_k_par[st] = ph;
          const int vs = kv % kVStages, vph = (kv / kVStages) & 1;
          if (!mbar_wait(bar_addr(sbase, VEMPTY + vs), vph ^ 1, abort_flag, p.wait_ns)) { ok = false; break; }
          mbar_expect_tx(bar_addr(sbase, VFULL + vs), kTileBytes + (kCkGlobal ? 512 : 0));
          for (int hf = 0; hf < kHalves; ++hf)
            tma_load_4d(sbase + kV + vs * kTile + hf * kHalf, &tm_v, bar_addr(sbase, VFULL + vs), hf * 64, U.hk,
                        n * 128, U.b);
          if (kCkGlobal)
            bulk_load(sbase + kCK + vs * 512, p.ck + ((size_t)U.b * (p.H / p.grp) + U.hk) * p.T_pad + n * 128, 512,
                      bar_addr(sbase, VFULL + vs));
          last_v_par[vs] = vph;
        }
        ++uidx;
      }
      {
        // Every exit, normal or aborted: the copies still in flight land before
        // the CTA's shared memory goes away (on the normal path they have landed).
        for (int s = 0; s < kKStages; ++s)
          if (last_k_par[s] >= 0) mbar_drain(bar_addr(sbase, KFULL + s), last_k_par[s]);
        for (int s = 0; s < kVStages; ++s)
          if (last_v_par[s] >= 0) mbar_drain(bar_addr(sbase, VFULL + s), last_v_par[s]);
        if (last_q_par >= 0) mbar_drain(bar_addr(sbase, QFULL), last_q_par);
      }
    } else if (warp == 9 && lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      constexpr uint32_t id_qk = idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t id_pv = idesc_bf16(128, kD, 0, 1);
      // Descriptor bases; every operand below is a base plus a constant byte offset.
      const uint64_t dQ_k = sdesc_sw128(sbase + kQ, 16, 1024), dK_k = sdesc_sw128(sbase + kK, 16, 1024);
      const uint64_t dV_m = sdesc_sw128(sbase + kV, kHalf, 1024);
      auto issue_s = [&](int k, int st) {
        const uint64_t qb = sdesc_add(dQ_k, k * kTile), kb = sdesc_add(dK_k, st * kTile);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
          mma_ss(tbase + 128 * k, sdesc_add(qb, off), sdesc_add(kb, off), id_qk, kk > 0);
        }
      };
      auto issue_pv = [&](int k, int st, bool acc) {
        const uint64_t vb = sdesc_add(dV_m, st * kTile);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tbase + 256 + 128 * k, tbase + 128 * k + kk * 8, sdesc_add(vb, kk * 2048), id_pv,
                 (acc || kk > 0) ? 1u : 0u);
      };
      uint32_t kv = 0, pcount[2] = {0, 0}, ounits[2] = {0, 0};
      int uidx = 0;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int u = unit_index(cta, r, G);
        if (u >= p.n_units) break;
        const Unit U = decode(p, u);
        if (!mbar_wait(bar_addr(sbase, kRope ? QREADY : QFULL), uidx & 1, abort_flag, p.wait_ns)) break;
        {
          const int st = kv % kKStages, ph = (kv / kKStages) & 1;
          if (!mbar_wait(bar_addr(sbase, KFULL + st), ph, abort_flag, p.wait_ns)) break;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 2; ++k)
            if (U.in(k, U.hi_u)) {
              issue_s(k, st);
              mma_commit(bar_addr(sbase, SFULL + k));
            }
          mma_commit(bar_addr(sbase, KEMPTY + st));
          // Q tiles are read only by the S products: after a unit's last one the
          // producer may load the next unit's Q
          if (U.N == 1) mma_commit(bar_addr(sbase, QEMPTY));
        }
        bool first_pv[2] = {true, true};
        for (int it = 0; it < U.N && ok; ++it) {
          const int n = U.hi_u - it;
          const uint32_t kvn = kv + it, kvx = kvn + 1;
          const int vsn = kvn % kVStages, vphn = (kvn / kVStages) & 1;
          const int stx = kvx % kKStages, phx = (kvx / kKStages) & 1;
          const bool has_next = it + 1 < U.N;
          if (!mbar_wait(bar_addr(sbase, VFULL + vsn), vphn, abort_flag, p.wait_ns)) { ok = false; break; }
          bool k_next_ready = false;
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            if (U.in(k, n)) {
              if (first_pv[k] && ounits[k] > 0 &&
                  !mbar_wait(bar_addr(sbase, OFREE + k), (ounits[k] - 1) & 1, abort_flag, p.wait_ns)) { ok = false; break; }
              if (!mbar_wait(bar_addr(sbase, PFULL + k), pcount[k] & 1, abort_flag, p.wait_ns)) { ok = false; break; }
              ++pcount[k];
              tc_fence_after();
              issue_pv(k, vsn, !first_pv[k]);
              first_pv[k] = false;
            }
            if (k == 1) mma_commit(bar_addr(sbase, VEMPTY + vsn));
            if (has_next && U.in(k, n - 1)) {
              if (!k_next_ready) {
                if (!mbar_wait(bar_addr(sbase, KFULL + stx), phx, abort_flag, p.wait_ns)) { ok = false; break; }
                k_next_ready = true;
              }
              tc_fence_after();
              issue_s(k, stx);
              mma_commit(bar_addr(sbase, SFULL + k));
            }
          }
          if (ok && has_next) mma_commit(bar_addr(sbase, KEMPTY + stx));
          if (ok && it + 2 == U.N) mma_commit(bar_addr(sbase, QEMPTY));
        }
        if (!ok) break;
#pragma unroll
        for (int k = 0; k < 2; ++k)
          if (U.valid[k]) {
            mma_commit(bar_addr(sbase, ODONE + k));
            ++ounits[k];
          }
        kv += U.N;
        ++uidx;
      }
      // Drain: every MMA issued by this thread completes before TMEM is freed.
      mma_commit(bar_addr(sbase, FINAL));
      mbar_drain(bar_addr(sbase, FINAL), 0);
    }
  } else {
    regs_inc<kRope ? kRegsHighPro : kRegsHigh>();
    // ------------------------------------------------------------ softmax warpgroups
    const int k = warp / 4;
    const int row = threadIdx.x & 127;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tbase + 128 * k + lane_off;
    const uint32_t tO = tbase + 256 + 128 * k + lane_off;
    const uint32_t qa = sbase + kQ + k * kTile;
    const float kLn2 = 0.69314718055994531f;
    uint32_t scount = 0, ecount = 0, kv = 0;
    int uidx = 0;
    bool ok = true;
    for (int r = 0; ok; ++r) {
      const int u = unit_index(cta, r, G);
      if (u >= p.n_units) break;
      const Unit U = decode(p, u);
      // this warpgroup's query tile, as scalars (no dynamic indexing into U)
      const bool validk = k ? U.valid[1] : U.valid[0];
      const int r0k = k ? U.r0[1] : U.r0[0];
      const int lok = k ? U.lo[1] : U.lo[0];
      const int hik = k ? U.hi[1] : U.hi[0];
      if (!validk) {
        kv += U.N;
        ++uidx;
        continue;
      }
      if (!__all_sync(0xffffffffu, mbar_wait(bar_addr(sbase, kRope ? QREADY : QFULL), uidx & 1, abort_flag, p.wait_ns)))
        break;
      const int i = r0k + row;
      // rq_i from this thread's own Q row in shared memory.
      float rq;
      {
        float ss[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int hf = 0; hf < kHalves; ++hf)
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 v = lds128(qa + hf * kHalf + sw128(row, c));
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float a = bf16lo(w4[e]), b2 = bf16hi(w4[e]);
              ss[e] = fmaf(a, a, ss[e]);
              ss[e] = fmaf(b2, b2, ss[e]);
            }
          }
        rq = rsqrtf((ss[0] + ss[1] + ss[2] + ss[3]) * kInvD + p.eps);
      }
      // l: row sum of the exponentials (gives lse); lr: row sum of the same values
      // rounded to bf16 as the P V product sees them (normalises O in the
      // fixed-offset path, so that o is an exact convex combination of v rows)
      float m = -INFINITY, l0 = 0.f, l1 = 0.f, lr0 = 0.f, lr1 = 0.f;
      bool first = true;
      for (int n = hik; n >= lok; --n) {
        const uint32_t kvn = kv + (U.hi_u - n);
        // key factors of this tile: in the ring (CKFULL) or loaded with V (VFULL).
        // They are normally ready before S, so this wait comes first and the one
        // on S is the last before the tile's work starts.
        constexpr int kSlots = kCkGlobal ? kVStages : kCkSlots;
        const int vsn = kvn % kSlots, vphn = (kvn / kSlots) & 1;
        if (!__all_sync(0xffffffffu,
                        mbar_wait(bar_addr(sbase, (kCkGlobal ? VFULL : CKFULL) + vsn), vphn, abort_flag, p.wait_ns))) {
          ok = false;
          break;
        }
        if (!__all_sync(0xffffffffu, mbar_wait(bar_addr(sbase, SFULL + k), scount & 1, abort_flag, p.wait_ns))) {
          ok = false;
          break;
        }
        ++scount;
        tc_fence_after();
        uint32_t s[128];
        tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
        tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
        tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&s[64]));
        tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&s[96]));
        tmem_wait_ld();
        const uint32_t ck_addr = sbase + kCK + vsn * 512;
        const int hi_c = i - n * 128;        // keys j <= hi_c are causal
        const int lo_c = i - p.w - n * 128;  // keys j >= lo_c are inside the window
        const bool edge = (n * 128 + 127 > r0k) || (r0k + 127 - n * 128 > p.w);
        if constexpr (kFixed) {
          // p_j = 2^(S_j ck_j rq - bound), in one pass, packed to bf16 pairs into
          // the S columns of TMEM; -inf outside the band on edge tiles
          const float negb = -p.bound;
          auto ppass = [&](auto masked_tag) {
            constexpr bool kMasked = decltype(masked_tag)::value;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t pk[16];
#pragma unroll
              for (int j4 = 0; j4 < 8; ++j4) {
                const int jb = 32 * c + 4 * j4;
                const float4 c4 = lds_f4(ck_addr + 4 * jb);
                float x[4];
                fmul2(x[0], x[1], __uint_as_float(s[jb]), __uint_as_float(s[jb + 1]), c4.x, c4.y);
                fmul2(x[2], x[3], __uint_as_float(s[jb + 2]), __uint_as_float(s[jb + 3]), c4.z, c4.w);
                if (kMasked) {
#pragma unroll
                  for (int e = 0; e < 4; ++e) x[e] = (jb + e > hi_c || jb + e < lo_c) ? -INFINITY : x[e];
                }
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                  float t0, t1;
                  ffma2(t0, t1, x[2 * h2], x[2 * h2 + 1], rq, rq, negb, negb);
                  const float p0 = ex2(t0), p1 = ex2(t1);
                  fadd2(l0, l1, p0, p1);
                  const uint32_t pp = pack_bf16(p0, p1);
                  add_bf16x2_f32(lr0, lr1, pp);
                  pk[2 * j4 + h2] = pp;
                }
              }
              tmem_st16(tS + 16 * c, pk);
            }
          };
          if (edge)
            ppass(std::integral_constant<bool, true>{});
          else
            ppass(std::integral_constant<bool, false>{});
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(bar_addr(sbase, PFULL + k));
          continue;
        }
        // x_j = S_j * ck_j (two at a time), masked to -inf outside the band on edge
        // tiles, with the running max taken three at a time
        float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
        auto xpass = [&](auto masked_tag) {
          constexpr bool kMasked = decltype(masked_tag)::value;
#pragma unroll
          for (int j4 = 0; j4 < 32; ++j4) {
            const float4 c4 = lds_f4(ck_addr + 16 * j4);
            float x[4];
            fmul2(x[0], x[1], __uint_as_float(s[4 * j4]), __uint_as_float(s[4 * j4 + 1]), c4.x, c4.y);
            fmul2(x[2], x[3], __uint_as_float(s[4 * j4 + 2]), __uint_as_float(s[4 * j4 + 3]), c4.z, c4.w);
            if (kMasked) {
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int j = 4 * j4 + e;
                x[e] = (j > hi_c || j < lo_c) ? -INFINITY : x[e];
              }
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) s[4 * j4 + e] = __float_as_uint(x[e]);
            if ((j4 & 1) == 0) {
              mx0 = fmax3(mx0, x[0], x[1]);
              mx1 = fmax3(mx1, x[2], x[3]);
            } else {
              mx2 = fmax3(mx2, x[0], x[1]);
              mx3 = fmax3(mx3, x[2], x[3]);
            }
          }
        };
        if (edge)
          xpass(std::integral_constant<bool, true>{});
        else
          xpass(std::integral_constant<bool, false>{});
        const float mrow = fmaxf(fmax3(mx0, mx1, mx2), mx3);
        const float mnew = fmaxf(m, mrow * rq);
        if (first) {
          m = mnew;
          first = false;
        } else {
          const bool need = mnew > m + 8.0f;
          if (__any_sync(0xffffffffu, need)) {
            const float alpha = need ? ex2(m - mnew) : 1.0f;
            if (need) {
              m = mnew;
              l0 *= alpha;
              l1 *= alpha;
            }
#pragma unroll 1
            for (int c = 0; c < kD / 32; ++c) {
              uint32_t ov[32];
              tmem_ld32(tO + 32 * c, ov);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; e += 2) {
                float a0, a1;
                fmul2(a0, a1, __uint_as_float(ov[e]), __uint_as_float(ov[e + 1]), alpha, alpha);
                ov[e] = __float_as_uint(a0);
                ov[e + 1] = __float_as_uint(a1);
              }
              tmem_st32(tO + 32 * c, ov);
            }
            tmem_wait_st();
          }
        }
        // p_j = 2^(x_j rq - m), packed to bf16 pairs into the S columns of TMEM
        const float negm = -m;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float t0, t1;
            ffma2(t0, t1, __uint_as_float(s[32 * c + 2 * e]), __uint_as_float(s[32 * c + 2 * e + 1]), rq, rq, negm,
                  negm);
            const float p0 = ex2(t0), p1 = ex2(t1);
            fadd2(l0, l1, p0, p1);
            pk[e] = pack_bf16(p0, p1);
          }
          tmem_st16(tS + 16 * c, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar_addr(sbase, PFULL + k));
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue
      if (!__all_sync(0xffffffffu, mbar_wait(bar_addr(sbase, ODONE + k), ecount & 1, abort_flag, p.wait_ns))) break;
      ++ecount;
      tc_fence_after();
      const float l = l0 + l1;
      const float inv = 1.0f / (kFixed ? lr0 + lr1 : l);
      const bool iv = i < p.T;
      __nv_bfloat16* orow = p.o + (((size_t)U.b * p.T + (iv ? i : 0)) * p.H + U.h) * kD;
#pragma unroll 1
      for (int c = 0; c < kD / 32; ++c) {
        uint32_t ov[32];
        tmem_ld32(tO + 32 * c, ov);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float a0, a1;
          fmul2(a0, a1, __uint_as_float(ov[2 * e]), __uint_as_float(ov[2 * e + 1]), inv, inv);
          pk[e] = pack_bf16(a0, a1);
        }
        if (iv) {
          stg32B(orow + 32 * c, pk, p.wide);
          stg32B(orow + 32 * c + 16, pk + 8, p.wide);
        }
      }
      tc_fence_before();
      mbar_arrive(bar_addr(sbase, OFREE + k));
      if (iv && p.lse) p.lse[(size_t)U.bh * p.T + i] = ((kFixed ? p.bound : m) + log2f(l)) * kLn2;
      kv += U.N;
      ++uidx;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

}  // namespace fwd
}  // namespace ar
